"""GPU parity of the causal-window decode step (lf_attn_decode) against the
oracle: the decode output of a sequence of length L equals row L-1 of the
oracle's causal forward over the first L positions (same dilation, window).
"""
import math

import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, n, r, dilation per head, lengths per sequence
    (2, 2, 300, 5, [1, 2], [300, 17]),
    (2, 3, 1100, 64, [1, 2, 3], [1, 1100]),
    (1, 2, 2100, 512, [1, 2], [2100]),
    (3, 1, 40, 0, [1], [40, 1, 7]),
]


@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_decode_matches_oracle_last_row(case, dtype):
    import torch
    B, H, n, r, dil, lens = CASES[case]
    wl = synth.custom("dec", B, H, n, r, dil, True, dtype, np.ones((B, n), np.int32), seed=100 + case)
    inp = synth.inputs_for(wl)
    q_full = inp["qs"]                     # the new token's query sits at row L-1
    lengths = np.asarray(lens, np.int32)
    q_new = np.stack([q_full[b, :, lengths[b] - 1] for b in range(B)])   # [B, H, 64]
    g = U.gpu_inputs(inp, dtype)
    q_dev = U.to_torch(np.ascontiguousarray(q_new), dtype)
    o = torch.empty_like(q_dev)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    p = L.make_params(B, H, n, r, dil, True, 0.0, {"f32": L.LF_F32, "bf16": L.LF_BF16, "f16": L.LF_F16}[dtype])
    L.lf_attn_decode(p, q_dev, g["ks"], g["vs"], torch.from_numpy(lengths).cuda(), o, lse)
    torch.cuda.synchronize()
    f = U.f64_inputs(inp, dtype)
    ref_o = np.zeros((B, H, 64))
    ref_l = np.zeros((B, H))
    for b in range(B):
        Lb = int(lengths[b])
        for h in range(H):
            oo, ll = oracle.fwd_head(r, dil[h], True, 1 / math.sqrt(64), np.ones(Lb, np.int32),
                                     f["qs"][b, h, :Lb], f["ks"][b, h, :Lb], f["vs"][b, h, :Lb],
                                     f["qs"][b, h, :Lb], f["ks"][b, h, :Lb], f["vs"][b, h, :Lb])
            ref_o[b, h] = oo[Lb - 1]
            ref_l[b, h] = ll[Lb - 1]
    U.compare("decode/o", U.to_f64(o), ref_o, dtype)
    U.compare_lse(U.to_f64(lse), ref_l, dtype)


def test_decode_requires_causal_and_handles_bad_lengths():
    import torch
    p = L.make_params(1, 1, 64, 4, None, False, 0.0, L.LF_BF16)
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    lens = torch.tensor([10], dtype=torch.int32, device="cuda")
    o = torch.empty((1, 1, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(L.LfError) as e:
        L.lf_attn_decode(p, o, x, x, lens, o)
    assert e.value.code == L.LF_ERR_INVALID
    p = L.make_params(2, 1, 64, 4, None, True, 0.0, L.LF_BF16)
    x = torch.ones((2, 1, 64, 64), dtype=torch.bfloat16, device="cuda")
    q = torch.ones((2, 1, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.full((2, 1, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((2, 1), dtype=torch.float32, device="cuda")
    L.lf_attn_decode(p, q, x, x, torch.tensor([0, 65], dtype=torch.int32, device="cuda"), o, lse)
    torch.cuda.synchronize()
    assert torch.all(o == 0) and torch.all(torch.isinf(lse))
