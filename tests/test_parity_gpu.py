"""GPU parity on small problems: the CUDA library (through its C ABI) against
the CPU oracle on the same seeded, dtype-rounded inputs.

Sizes span several 128-row tiles and a ragged tail; the cases cover the edge
structure of the method: tiny and large windows, dilation 1..3 per head,
causal windows, padding tails, global tokens at the ends / adjacent / inside
the window, more global tokens than one key tile, sequences with no local
token, a window wider than the sequence, and n = 1.
Forward (o, lse), pair counts (exact), the pattern itself (exact) and the
backward (six gradients) are all compared.
"""
import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu


def _mask(B, n, lengths=None, globals_=None):
    m = np.ones((B, n), np.int32)
    for b in range(B):
        if lengths is not None:
            m[b, lengths[b]:] = 0
        if globals_ is not None:
            for g in globals_[b]:
                m[b, g] = 2
    return m


def _cases():
    rng = np.random.default_rng(5)
    many = sorted(rng.choice(np.arange(1, 600), size=150, replace=False).tolist())
    C = {}
    C["r64_g0"] = dict(B=2, H=2, n=700, r=64, dil=[1, 1], causal=False,
                       mask=_mask(2, 700, globals_=[[0], [0]]))
    C["r1_local"] = dict(B=1, H=2, n=300, r=1, dil=[1, 1], causal=False, mask=_mask(1, 300))
    C["r256_pad_glob"] = dict(B=2, H=3, n=1000, r=256, dil=[1, 1, 1], causal=False,
                              mask=_mask(2, 1000, lengths=[1000, 777], globals_=[[0, 5, 400], [0, 770]]))
    C["dilated_123"] = dict(B=1, H=4, n=900, r=40, dil=[1, 2, 3, 1], causal=False,
                            mask=_mask(1, 900, globals_=[[3, 500]]))
    C["causal_dil"] = dict(B=1, H=2, n=650, r=100, dil=[1, 2], causal=True, mask=_mask(1, 650))
    C["causal_pad"] = dict(B=2, H=1, n=513, r=63, dil=[1], causal=True,
                           mask=_mask(2, 513, lengths=[513, 300]))
    C["many_globals"] = dict(B=1, H=2, n=640, r=16, dil=[1, 2], causal=False,
                             mask=_mask(1, 640, globals_=[many]))
    C["globals_edges"] = dict(B=1, H=2, n=400, r=8, dil=[1, 1], causal=False,
                              mask=_mask(1, 400, globals_=[[0, 1, 2, 10, 395, 398, 399]]))
    m = np.zeros((2, 256), np.int32)
    m[0, [0, 100, 255]] = 2
    m[1, :] = 0
    C["no_local_rows"] = dict(B=2, H=1, n=256, r=32, dil=[1], causal=False, mask=m)
    C["window_ge_n"] = dict(B=1, H=2, n=200, r=300, dil=[1, 3], causal=False,
                            mask=_mask(1, 200, globals_=[[7]]))
    C["n1"] = dict(B=1, H=1, n=1, r=4, dil=[1], causal=False, mask=_mask(1, 1))
    # a causal window wider than the sequence: full causal (decoder) self-attention
    C["causal_dense"] = dict(B=1, H=2, n=600, r=1000, dil=[1, 1], causal=True, mask=_mask(1, 600))
    # 11 residue sub-sequences (1 + 2 + 8): more tensor maps than a small
    # parameter block holds; the tensor-core kernels take it (no fallback)
    C["dil_1_2_8"] = dict(B=1, H=3, n=1100, r=40, dil=[1, 2, 8], causal=False,
                          mask=_mask(1, 1100, globals_=[[0, 555]]))
    # large scores (inputs N(0, 3^2) / N(0, 4^2)): row sums leave the range the
    # running reference allows, so the tensor-core softmax redoes tiles with
    # the row's tile max (overflow side) and, with two keys per row, with
    # all-tiny tiles (underflow side)
    C["hot_scores"] = dict(B=1, H=2, n=600, r=64, dil=[1, 2], causal=False,
                           mask=_mask(1, 600, globals_=[[0, 300]]), in_scale=3.0)
    C["hot_causal_r1"] = dict(B=1, H=1, n=300, r=1, dil=[1], causal=True, mask=_mask(1, 300),
                              in_scale=4.0)
    return C


CASES = _cases()
KERNELS = [("f32", L.LF_KERNEL_SIMT), ("bf16", L.LF_KERNEL_SIMT), ("f16", L.LF_KERNEL_SIMT),
           ("bf16", L.LF_KERNEL_TC), ("f16", L.LF_KERNEL_TC), ("f32", L.LF_KERNEL_AUTO)]


def _setup(name, dtype, kernel, seed=11, backward=False):
    c = CASES[name]
    wl = synth.custom(name, c["B"], c["H"], c["n"], c["r"], c["dil"], c["causal"], dtype, c["mask"],
                      seed=seed, in_scale=c.get("in_scale", 1.0), backward=backward)
    inp = synth.inputs_for(wl)
    if c.get("in_scale", 1.0) != 1.0:
        # large scores, unit-scale values: O stays within the absolute tolerance
        for kname in ("vs", "vg"):
            inp[kname] = synth.round_to(synth.as_float64(inp[kname], dtype) / c["in_scale"], dtype)
    ng = int((c["mask"] == 2).sum(axis=1).max())
    att = L.LongformerAttention(c["B"], c["H"], c["n"], c["r"], c["dil"], c["causal"], dtype=dtype,
                                max_global=ng, kernel=kernel)
    return c, wl, inp, att


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_forward_default_max_global_long_sequence(dtype):
    """max_global left at its default (-1: room for n global rows) on a
    sequence longer than 8192: the global list no longer fits the fused mask
    pass + gather kernel, so the separate mask pass and gather kernels run."""
    n = 8500
    m = _mask(1, n, globals_=[[0, 4000, n - 1]])
    wl = synth.custom("long_default_g", 1, 1, n, 32, [1], False, dtype, m, seed=23)
    inp = synth.inputs_for(wl)
    att = L.LongformerAttention(1, 1, n, 32, [1], False, dtype=dtype, kernel=L.LF_KERNEL_TC)
    g = U.gpu_inputs(inp, dtype)
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    att.status()
    f = U.f64_inputs(inp, dtype)
    ro, rl = oracle.fwd(32, [1], False, U.scale_of(wl), inp["mask"], f["qs"], f["ks"], f["vs"],
                        f["qg"], f["kg"], f["vg"])
    U.compare("long_default_g/o", U.to_f64(o), ro, dtype)
    U.compare_lse(U.to_f64(lse), rl, dtype)


@pytest.mark.parametrize("dtype,kernel", KERNELS)
@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_parity(name, dtype, kernel):
    c, wl, inp, att = _setup(name, dtype, kernel)
    g = U.gpu_inputs(inp, dtype)
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    att.status()
    f = U.f64_inputs(inp, dtype)
    scale = U.scale_of(wl)
    ro, rl = oracle.fwd(c["r"], c["dil"], c["causal"], scale, inp["mask"], f["qs"], f["ks"], f["vs"],
                        f["qg"], f["kg"], f["vg"])
    U.compare(name + "/o", U.to_f64(o), ro, dtype)
    U.compare_lse(U.to_f64(lse), rl, dtype)


@pytest.mark.parametrize("name", sorted(CASES))
def test_pair_counts_and_pattern_exact(name):
    c, wl, inp, att = _setup(name, "bf16", L.LF_KERNEL_AUTO)
    import torch
    mask = torch.from_numpy(inp["mask"]).cuda()
    got = att.count_pairs(mask).cpu().numpy()
    att.status()
    ref = oracle.counts(c["r"], c["dil"], c["causal"], inp["mask"], c["H"])
    assert np.array_equal(got, ref), (got, ref)
    dump = att.mask_dump(mask).cpu().numpy()
    for b in range(c["B"]):
        for h in range(c["H"]):
            A = oracle.pattern(c["n"], c["r"], c["dil"][h], c["causal"], inp["mask"][b])
            assert np.array_equal(dump[b, h], A), (b, h)


# Unit-scale cases take the fixed bounds below.  On the large-score cases
# (nearly one-hot rows) the 16-bit error is set by the cancellation in
# dS = p (dP - D) and scales with the inputs; those take the elementwise
# first-order bound of lfutil.bwd_error_bound instead (test below).
BWD_CASES = sorted(k for k, c in CASES.items() if c.get("in_scale", 1.0) == 1.0)
HOT_CASES = sorted(k for k, c in CASES.items() if c.get("in_scale", 1.0) != 1.0)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("name", BWD_CASES)
def test_backward_parity(name, dtype):
    c, wl, inp, att = _setup(name, dtype, L.LF_KERNEL_AUTO, backward=True)
    g = U.gpu_inputs(inp, dtype)
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    grads = att.bwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse, g["do"])
    att.status(bwd=True)
    f = U.f64_inputs(inp, dtype)
    # the oracle sees the same rounded dO
    ref = oracle.bwd(c["r"], c["dil"], c["causal"], U.scale_of(wl), inp["mask"], f["qs"], f["ks"],
                     f["vs"], f["qg"], f["kg"], f["vg"], f["do"])
    for k, nm in enumerate(["dq_s", "dk_s", "dv_s", "dq_g", "dk_g", "dv_g"]):
        U.compare(name + "/" + nm, U.to_f64(grads[k]), ref[k], dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("name", HOT_CASES)
def test_backward_parity_large_scores(name, dtype):
    """Backward on Q, K at 3x / 4x scale: every gradient element within the
    derived first-order bound (dS and P rounded to the format, D from the
    rounded forward output) plus the rounding of the stored gradient."""
    c, wl, inp, att = _setup(name, dtype, L.LF_KERNEL_TC, backward=True)
    g = U.gpu_inputs(inp, dtype)
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    grads = att.bwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse, g["do"])
    att.status(bwd=True)
    f = U.f64_inputs(inp, dtype)
    scale = U.scale_of(wl)
    ref = oracle.bwd(c["r"], c["dil"], c["causal"], scale, inp["mask"], f["qs"], f["ks"], f["vs"],
                     f["qg"], f["kg"], f["vg"], f["do"])
    bound = U.bwd_error_bound(c, scale, inp["mask"], f, dtype)
    for k, nm in enumerate(["dq_s", "dk_s", "dv_s", "dq_g", "dk_g", "dv_g"]):
        U.compare_bound(name + "/" + nm, U.to_f64(grads[k]), ref[k], bound[k], dtype, factor=1.0)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_tensor_core_many_residues_fwd_bwd(dtype):
    """Dilations 1, 2, 8 on the tensor-core kernels, asked for explicitly:
    both run it (the shape is inside their parameter blocks) and match."""
    name = "dil_1_2_8"
    c, wl, inp, att = _setup(name, dtype, L.LF_KERNEL_TC, backward=True)
    g = U.gpu_inputs(inp, dtype)
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    att.status()
    grads = att.bwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"], o, lse, g["do"])
    att.status(bwd=True)
    f = U.f64_inputs(inp, dtype)
    scale = U.scale_of(wl)
    ro, rl = oracle.fwd(c["r"], c["dil"], c["causal"], scale, inp["mask"], f["qs"], f["ks"], f["vs"],
                        f["qg"], f["kg"], f["vg"])
    U.compare(name + "/o", U.to_f64(o), ro, dtype)
    U.compare_lse(U.to_f64(lse), rl, dtype)
    ref = oracle.bwd(c["r"], c["dil"], c["causal"], scale, inp["mask"], f["qs"], f["ks"], f["vs"],
                     f["qg"], f["kg"], f["vg"], f["do"])
    for k, nm in enumerate(["dq_s", "dk_s", "dv_s", "dq_g", "dk_g", "dv_g"]):
        U.compare(name + "/" + nm, U.to_f64(grads[k]), ref[k], dtype)


def test_device_status_flags():
    """Device-side input problems land in the status word (no fault)."""
    import torch
    n = 256
    m = np.ones((1, n), np.int32)
    m[0, [0, 9, 70]] = 2
    att = L.LongformerAttention(1, 1, n, 8, dtype="bf16", max_global=2)   # 3 > 2 globals
    x = torch.zeros((1, 1, n, 64), dtype=torch.bfloat16, device="cuda")
    att.fwd(x, x, x, x, x, x, torch.from_numpy(m).cuda())
    with pytest.raises(L.LfError) as e:
        att.status()
    assert e.value.code == L.LF_ERR_DEVICE_INPUT
    att.status()   # cleared by the read
    m2 = m.copy()
    m2[0, 5] = 7
    att2 = L.LongformerAttention(1, 1, n, 8, dtype="bf16", max_global=8)
    att2.fwd(x, x, x, x, x, x, torch.from_numpy(m2).cuda())
    with pytest.raises(L.LfError) as e:
        att2.status()
    assert e.value.code == L.LF_ERR_DEVICE_INPUT
    att3 = L.LongformerAttention(1, 1, n, 8, causal=True, dtype="bf16", max_global=8)
    att3.fwd(x, x, x, x, x, x, torch.from_numpy(m).cuda())
    with pytest.raises(L.LfError) as e:
        att3.status()
    assert e.value.code == L.LF_ERR_UNSUPPORTED
