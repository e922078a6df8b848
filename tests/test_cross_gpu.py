"""Parity of the LED decoder cross-attention (lf_attn_cross_fwd) with the
oracle's dense cross-attention, element by element, on the same rounded
inputs.  Tolerances as for the self-attention forward (tests/lfutil.py)."""
import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu


def _run(B, H, Lq, Lk, dtype, kmask, seed, heads=None):
    import torch
    q = synth.tensor(seed, "qs", (B, H, Lq, 64), dtype)
    k = synth.tensor(seed, "ks", (B, H, Lk, 64), dtype)
    v = synth.tensor(seed, "vs", (B, H, Lk, 64), dtype)
    p = L.make_cross_params(B, H, Lq, Lk, L._DT[dtype])
    ws = L.cross_workspace(p)
    tq, tk, tv = (U.to_torch(a, dtype) for a in (q, k, v))
    o = torch.empty_like(tq)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device="cuda")
    km = None if kmask is None else torch.from_numpy(kmask).cuda()
    L.lf_attn_cross_fwd(p, tq, tk, tv, km, o, lse, ws)
    L.lf_attn_status(ws)
    ro, rl = oracle.cross(1.0 / 8.0, kmask, *(synth.as_float64(a, dtype) for a in (q, k, v)), heads=heads)
    return U.to_f64(o), U.to_f64(lse), ro, rl


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_cross_ragged_with_key_padding(dtype):
    B, Lk = 2, 1000
    km = np.ones((B, Lk), np.int32)
    km[1, 800:] = 0
    km[0, [5, 77, 999]] = 0
    o, lse, ro, rl = _run(B, 3, 300, Lk, dtype, km, 51)
    U.compare("cross/o", o, ro, dtype)
    U.compare_lse(lse, rl, dtype)


@pytest.mark.parametrize("Lq,Lk", [(1, 777), (129, 128), (64, 4097)])
def test_cross_shapes_without_mask(Lq, Lk):
    o, lse, ro, rl = _run(1, 2, Lq, Lk, "bf16", None, 52 + Lq)
    U.compare("cross/o", o, ro, "bf16")
    U.compare_lse(lse, rl, "bf16")


def test_cross_sequence_with_no_valid_key():
    km = np.ones((2, 300), np.int32)
    km[1, :] = 0
    o, lse, ro, rl = _run(2, 2, 100, 300, "bf16", km, 53)
    assert np.all(o[1] == 0) and np.all(np.isneginf(lse[1]))
    U.compare("cross/o", o, ro, "bf16")
    U.compare_lse(lse, rl, "bf16")


def test_cross_led_decoder_shape_sampled_heads():
    """The LED shape of the pages: 1024 decoder positions against a 16K
    encoder output, 16 heads, two sequences (the second padded to 12000
    keys); two heads compared in full."""
    B, H, Lq, Lk = 2, 16, 1024, 16384
    km = np.ones((B, Lk), np.int32)
    km[1, 12000:] = 0
    heads = [(0, 0), (1, 15)]
    o, lse, ro, rl = _run(B, H, Lq, Lk, "bf16", km, 54, heads=heads)
    for b, h in heads:
        U.compare("cross/o[%d,%d]" % (b, h), o[b, h], ro[b, h], "bf16")
        U.compare_lse(lse[b, h], rl[b, h], "bf16")
