"""Helpers shared by the tests: move synth storage arrays to torch, run the
CUDA library through its C ABI, run the oracle on the same rounded inputs,
and compare with the stated tolerances."""
from __future__ import annotations

import math
import numpy as np

from sparse_sliding_window_b200 import synth

# tolerances (max-abs for f32; max-abs + relative L2 for bf16/f16)
TOL = {"f32": dict(max_abs=1e-4, rel_l2=1e-5),
       "bf16": dict(max_abs=2e-2, rel_l2=1e-2),
       "f16": dict(max_abs=2e-2, rel_l2=1e-2)}
LSE_TOL = {"f32": 1e-4, "bf16": 2e-3, "f16": 2e-3}


def to_torch(arr: np.ndarray, dtype: str, device="cuda"):
    import torch
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr))
    return t.to(device)


def to_f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def f64_inputs(inp: dict, dtype: str) -> dict:
    return {k: synth.as_float64(v, dtype) for k, v in inp.items() if k not in ("mask", "dilation")}


def gpu_inputs(inp: dict, dtype: str, device="cuda") -> dict:
    import torch
    out = {k: to_torch(v, dtype, device) for k, v in inp.items() if k not in ("mask", "dilation")}
    out["mask"] = torch.from_numpy(inp["mask"]).to(device)
    return out


def compare(name: str, got: np.ndarray, ref: np.ndarray, dtype: str, max_abs=None, rel_l2=None):
    """Assert closeness over the entries where ref is defined (not NaN)."""
    sel = ~np.isnan(ref)
    g, r = got[sel], ref[sel]
    assert np.all(np.isfinite(g)), name + ": non-finite output"
    err = np.abs(g - r)
    mabs = float(err.max()) if err.size else 0.0
    rl2 = float(np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)) if err.size else 0.0
    tol = TOL[dtype]
    ma = tol["max_abs"] if max_abs is None else max_abs
    rl = tol["rel_l2"] if rel_l2 is None else rel_l2
    assert mabs <= ma, "%s: max-abs %.3e > %.1e (rel-L2 %.3e)" % (name, mabs, ma, rl2)
    # relative L2 only where the reference is not (numerically) zero: e.g. the
    # dQ / dK of a row that attends only itself are exactly zero
    if dtype != "f32" and np.linalg.norm(r) > 1e-6 * max(1, r.size) ** 0.5:
        assert rl2 <= rl, "%s: rel-L2 %.3e > %.1e (max-abs %.3e)" % (name, rl2, rl, mabs)
    return mabs, rl2


def compare_lse(got: np.ndarray, ref: np.ndarray, dtype: str):
    sel = ~np.isnan(ref)
    g, r = got[sel], ref[sel]
    inf_r = np.isinf(r)
    assert np.array_equal(np.isinf(g) & (g < 0), inf_r), "lse: -inf rows differ"
    e = np.abs(g[~inf_r] - r[~inf_r])
    m = float(e.max()) if e.size else 0.0
    assert m <= LSE_TOL[dtype], "lse max-abs %.3e > %.1e" % (m, LSE_TOL[dtype])
    return m


def scale_of(wl) -> float:
    return 1.0 / math.sqrt(wl.head_dim)
