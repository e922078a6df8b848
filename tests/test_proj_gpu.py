"""Parity of the projection GEMM (include/lf_proj.h) against the oracle's
double-precision affine map, element by element.

Tolerance, from the arithmetic: the products of two 16-bit values are exact
in fp32 and the tensor cores sum them in fp32, so before rounding the error
is at most K * 2^-24 * sum_k |x_k w_k| (first order, any summation order);
the bias is added in fp32 and the result rounded once to the 16-bit format,
an error of at most u |y| with u = 2^-8 (bf16) / 2^-11 (f16), taken here as
the format's full relative spacing.  Every element must satisfy
|got - ref| <= u |ref| + K 2^-24 sum_k |x_k| |w_k| + 1e-6.
"""
import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu

U16 = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}


def _rand(seed, name, shape, dtype, scale=1.0):
    return synth.tensor(seed, name, shape, dtype, scale)


def _bound(x64, w64, ref, dtype):
    K = x64.shape[-1]
    acc = oracle.linear(np.abs(x64), np.abs(w64))
    return U16[dtype] * np.abs(ref) + K * 2.0 ** -24 * acc + 1e-6


def _assert_within(name, got, ref, bound):
    err = np.abs(got - ref)
    assert np.all(np.isfinite(got)), name + ": non-finite"
    worst = float((err / bound).max())
    k = np.unravel_index(int(np.argmax(err / bound)), err.shape)
    assert worst <= 1.0, "%s: error %.3e above bound %.3e at %s" % (name, err[k], bound[k], k)


def _inputs(B, n, H, nproj, dtype, seed, bias=True):
    D = H * 64
    x = _rand(seed, "x", (B, n, D), dtype)
    w = _rand(seed, "w", (nproj * D, D), dtype, scale=D ** -0.5)
    b = _rand(seed, "b", (nproj * D,), dtype, scale=0.1) if bias else None
    return x, w, b


@pytest.mark.parametrize("dtype,B,n,H,nproj,bias", [
    ("bf16", 1, 4096, 12, 5, True),     # longformer-base shape: Q_s, K_s, V_s, K_g, V_g
    ("f16", 2, 300, 4, 3, False),       # ragged last row block, two sequences, no bias
    ("bf16", 2, 129, 8, 1, True),       # one row past a block
])
def test_input_projection_parity(dtype, B, n, H, nproj, bias):
    import torch
    D = H * 64
    x, w, b = _inputs(B, n, H, nproj, dtype, 31 + n, bias)
    p = L.make_proj_params(B, n, H, L._DT[dtype])
    ws = L.proj_workspace(p, 0)
    outs = [torch.empty((B, H, n, 64), dtype=torch.bfloat16 if dtype == "bf16" else torch.float16,
                        device="cuda") for _ in range(nproj)]
    L.lf_proj_in(p, U.to_torch(x, dtype), U.to_torch(w, dtype), None if b is None else U.to_torch(b, dtype),
                 outs, ws)
    L.lf_attn_status(ws)
    x64, w64 = synth.as_float64(x, dtype), synth.as_float64(w, dtype)
    b64 = None if b is None else synth.as_float64(b, dtype)
    ref = oracle.linear(x64, w64, b64)             # [B, n, nproj*D]
    bound = _bound(x64, w64, ref, dtype)
    for k in range(nproj):
        got = U.to_f64(outs[k]).transpose(0, 2, 1, 3).reshape(B, n, D)
        sl = slice(k * D, (k + 1) * D)
        _assert_within("proj%d" % k, got, ref[..., sl], bound[..., sl])


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_global_row_projection_only_at_global_tokens(dtype):
    """Q_g at the global tokens of the attention mask only: those rows match
    the oracle, every other row keeps what the buffer held."""
    import torch
    B, n, H = 2, 700, 12
    D = H * 64
    x, w, b = _inputs(B, n, H, 1, dtype, 77)
    m = np.ones((B, n), np.int32)
    g0 = list(range(0, 65))
    g1 = [3, 350, 699]
    m[0, g0] = 2
    m[1, g1] = 2
    m[1, 600:] = 0
    m[1, 699] = 2
    p = L.make_proj_params(B, n, H, L._DT[dtype])
    ws = L.proj_workspace(p, 65)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    out = torch.full((B, H, n, 64), 7.0, dtype=tdt, device="cuda")
    L.lf_proj_in(p, U.to_torch(x, dtype), U.to_torch(w, dtype), U.to_torch(b, dtype), [out], ws,
                 rows_mask=torch.from_numpy(m).cuda(), rows_code=2, max_rows=65)
    L.lf_attn_status(ws)
    x64, w64, b64 = (synth.as_float64(a, dtype) for a in (x, w, b))
    ref = oracle.linear(x64, w64, b64)
    bound = _bound(x64, w64, ref, dtype)
    got = U.to_f64(out).transpose(0, 2, 1, 3).reshape(B, n, D)
    for bb, rows in ((0, g0), (1, g1)):
        _assert_within("qg[%d]" % bb, got[bb, rows], ref[bb, rows], bound[bb, rows])
        other = np.setdiff1d(np.arange(n), rows)
        assert np.all(got[bb, other] == 7.0), "rows outside the selection were written"


def test_selected_rows_above_max_rows_flagged():
    import torch
    B, n, H = 1, 300, 4
    x, w, b = _inputs(B, n, H, 1, "bf16", 5)
    m = np.ones((B, n), np.int32)
    m[0, :10] = 2
    p = L.make_proj_params(B, n, H, L.LF_BF16)
    ws = L.proj_workspace(p, 4)
    out = torch.zeros((B, H, n, 64), dtype=torch.bfloat16, device="cuda")
    L.lf_proj_in(p, U.to_torch(x, "bf16"), U.to_torch(w, "bf16"), U.to_torch(b, "bf16"), [out], ws,
                 rows_mask=torch.from_numpy(m).cuda(), rows_code=2, max_rows=4)
    with pytest.raises(L.LfError) as e:
        L.lf_attn_status(ws)
    assert e.value.code == L.LF_ERR_DEVICE_INPUT
    # the first max_rows selected rows are still projected
    ref = oracle.linear(*(synth.as_float64(a, "bf16") for a in (x, w, b)))
    got = U.to_f64(out).transpose(0, 2, 1, 3).reshape(B, n, H * 64)
    bound = _bound(synth.as_float64(x, "bf16"), synth.as_float64(w, "bf16"), ref, "bf16")
    _assert_within("first rows", got[0, :4], ref[0, :4], bound[0, :4])
    assert np.all(got[0, 4:] == 0)


@pytest.mark.parametrize("dtype,B,n,H", [("bf16", 1, 4096, 12), ("f16", 2, 333, 8)])
def test_output_projection_parity(dtype, B, n, H):
    import torch
    D = H * 64
    o = _rand(90 + n, "o", (B, H, n, 64), dtype)
    w = _rand(90 + n, "wo", (D, D), dtype, scale=D ** -0.5)
    b = _rand(90 + n, "bo", (D,), dtype, scale=0.1)
    p = L.make_proj_params(B, n, H, L._DT[dtype])
    ws = L.proj_workspace(p, 0)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    y = torch.empty((B, n, D), dtype=tdt, device="cuda")
    L.lf_proj_out(p, U.to_torch(o, dtype), U.to_torch(w, dtype), U.to_torch(b, dtype), y, ws)
    L.lf_attn_status(ws)
    # heads concatenated: input feature h*64 + c of token t is o[b, h, t, c]
    o64 = synth.as_float64(o, dtype).transpose(0, 2, 1, 3).reshape(B, n, D)
    w64, b64 = synth.as_float64(w, dtype), synth.as_float64(b, dtype)
    ref = oracle.linear(o64, w64, b64)
    _assert_within("y", U.to_f64(y), ref, _bound(o64, w64, ref, dtype))
