"""lf_attn_fwd_noalloc: the forward for callers that cannot allocate device
memory (a plugin that only receives buffers from its host application, or
code that must not call cudaMalloc while it runs).  Its scratch is a fixed
array inside the library, so the test checks that two calls in a row on that
shared array -- with different masks, shapes and inputs -- match the regular
workspace entry point within the tolerances of the other parity tests, and
that a problem too large for the array is refused up front.

The array also holds the call's device status word, read through
lf_attn_status_noalloc: a mask value outside {0, 1, 2} must come back as
LF_ERR_DEVICE_INPUT there (the read clears the word), and the next good call
must come back clean.  Free device memory is compared around the calls: the
entry point exists so that nothing is allocated, so it must not drop.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test.
"""
import numpy as np
import pytest

from sparse_sliding_window_b200 import build as lfbuild
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu


def _case(B, H, n, r, dil, mask, seed, dtype="bf16"):
    import torch
    wl = synth.custom("noalloc", B, H, n, r, dil, False, dtype, mask, seed=seed)
    inp = synth.inputs_for(wl)
    g = U.gpu_inputs(inp, dtype)
    ng = int((mask == 2).sum(axis=1).max())
    p = L.make_params(B, H, n, r, dil, False, 0.0, {"bf16": L.LF_BF16, "f16": L.LF_F16}[dtype], ng)
    ws = L.workspace(p, False)
    o_ref = torch.empty_like(g["qs"])
    lse_ref = torch.empty(g["qs"].shape[:3], dtype=torch.float32, device="cuda")
    L.lf_attn_fwd(p, g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o_ref, lse_ref, ws)
    L.lf_attn_status(ws)
    return p, g, o_ref, lse_ref


def test_noalloc_matches_workspace_forward_two_calls():
    import torch
    lfbuild.build()
    L.load()
    m1 = np.ones((1, 1000), np.int32)
    m1[0, [0, 5, 400]] = 2
    m2 = np.ones((2, 700), np.int32)
    m2[0, 0] = 2
    m2[1, 500:] = 0
    m2[1, [3, 90]] = 2
    cases = [(1, 3, 1000, 64, [1, 2, 1], m1, 21, "bf16"), (2, 2, 700, 100, [1, 1], m2, 22, "f16")]
    prepared = [_case(*c) for c in cases]
    outs = [(torch.full_like(o_ref, float("nan")), torch.full_like(lse_ref, float("nan")))
            for _, _, o_ref, lse_ref in prepared]
    # warm-up calls: the library's device code (and with it the static array)
    # may be loaded lazily, kernel by kernel, on first use
    for (p, g, _, _), (o, lse) in zip(prepared, outs):
        L.lf_attn_fwd_noalloc(p, g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse)
        L.lf_attn_status_noalloc()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for (p, g, _, _), (o, lse) in zip(prepared, outs):   # two calls in a row on the shared scratch
        o.fill_(float("nan"))
        lse.fill_(float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        L.lf_attn_fwd_noalloc(p, g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse)
        L.lf_attn_status_noalloc()
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free_before  # nothing allocated by the call
    assert torch.cuda.mem_get_info()[0] == free0
    for (p, g, o_ref, lse_ref), (o, lse), c in zip(prepared, outs, cases):
        dt = c[-1]
        U.compare("noalloc/o", U.to_f64(o), U.to_f64(o_ref), dt)
        U.compare_lse(U.to_f64(lse), U.to_f64(lse_ref), dt)


def test_noalloc_status_reports_device_input_errors_then_clears():
    import torch
    lfbuild.build()
    L.load()
    m = np.ones((1, 500), np.int32)
    m[0, 0] = 2
    p, g, o_ref, lse_ref = _case(1, 2, 500, 32, [1, 1], m, 31)
    bad = g["mask"].clone()
    bad[0, 123] = 3                      # not a mask code: only the device sees it
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    L.lf_attn_fwd_noalloc(p, g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], bad, o, lse)
    with pytest.raises(L.LfError) as e:
        L.lf_attn_status_noalloc()
    assert e.value.code == L.LF_ERR_DEVICE_INPUT
    # the next good call starts from a clear status word and matches
    L.lf_attn_fwd_noalloc(p, g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse)
    L.lf_attn_status_noalloc()
    torch.cuda.synchronize()
    U.compare("noalloc/o after error", U.to_f64(o), U.to_f64(o_ref), "bf16")
    U.compare_lse(U.to_f64(lse), U.to_f64(lse_ref), "bf16")


def test_noalloc_refuses_problems_larger_than_its_scratch():
    import torch
    lfbuild.build()
    lib = L.load()
    p = L.make_params(8, 16, 65536, 256, None, False, 0.0, L.LF_BF16, max_global=65536)
    assert L.lf_attn_workspace_size(p, False) > L.LF_STATIC_WORKSPACE_BYTES
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LfError) as e:
        L.lf_attn_fwd_noalloc(p, x, x, x, x, x, x, x, x, None)
    assert e.value.code == L.LF_ERR_UNSUPPORTED
    assert b"static scratch" in lib.lf_attn_last_error()
