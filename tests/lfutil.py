"""Helpers shared by the tests: move synth storage arrays to torch, run the
CUDA library through its C ABI, run the oracle on the same rounded inputs,
and compare with the stated tolerances."""
from __future__ import annotations

import math
import numpy as np

import oracle
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


# unit roundoff of the 16-bit formats (round to nearest even)
UNIT_ROUNDOFF = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11}


def bwd_error_bound(c: dict, scale: float, mask: np.ndarray, f: dict, dtype: str,
                    lam: float = 6.0) -> list:
    """Elementwise error bound of the 16-bit backward for the six gradients
    (dQ_s, dK_s, dV_s, dQ_g, dK_g, dV_g), from the oracle's probabilities
    and forward.  Per attended pair (i, j) of row i (keys K, V and query q_i
    of the row's kind: global rows use the _g projections, local rows the
    _s ones), with u the format's unit roundoff:

      dP_ij = dO_i . V_j,  D_i = sum_j p_ij dP_ij,  dS_ij = p_ij (dP_ij - D_i)

    The error comes from roundings to the 16-bit format (fp32 accumulation
    and the exponent's error, relative ~1e-6 from the saved lse, are far
    below u), each an independent round-to-nearest error of zero mean and
    at most u |x|, so of variance <= (u x)^2 / 3:

    * D is formed from the rounded forward output O: O_id carries the
      rounding of o_id and of each p_ij in P.V, so
      var(dD_i) = sum_d dO_id^2 u^2 (o_id^2 + sum_j p_ij^2 V_jd^2) / 3.
      dD_i shifts every dS_ij of its row by -p_ij dD_i: dQ_i moves by
      -scale dD_i sum_j p_ij K_j, dK_j by -scale sum_i p_ij dD_i q_i;
    * dS (and P, for dV = P^T dO) is rounded before the tensor-core
      products: dQ_i moves by scale sum_j e_ij K_j with var(e_ij) =
      (u dS_ij)^2 / 3, and so on.

    The bound is lam standard deviations of the sum (probabilistic rounding
    error analysis in the manner of Higham and Mary); lam = 6.  The caller
    adds the rounding of the stored gradient, u |grad|."""
    u = UNIT_ROUNDOFF[dtype]
    B, H, n = c["B"], c["H"], c["n"]
    var = [np.zeros_like(f[k]) for k in ("qs", "ks", "vs", "qg", "kg", "vg")]
    for b in range(B):
        m = mask[b]
        for h in range(H):
            d = int(c["dil"][h])
            qs, ks, vs, qg, kg, vg, dO = (f[k][b, h] for k in ("qs", "ks", "vs", "qg", "kg", "vg", "do"))
            o, _ = oracle.fwd_head(c["r"], d, c["causal"], scale, m, qs, ks, vs, qg, kg, vg)
            for i in range(n):
                if m[i] == 0:
                    continue
                p = oracle.probs_row(i, c["r"], d, c["causal"], scale, m, qs, ks, qg, kg)
                glob = m[i] == 2
                K, V, qi = (kg, vg, qg[i]) if glob else (ks, vs, qs[i])
                dP = V @ dO[i]
                D = p @ dP
                dS = p * (dP - D)
                var_dD = u * u / 3.0 * ((dO[i] ** 2) @ (o[i] ** 2 + (p ** 2) @ (V ** 2)))
                iq, ik, iv = (3, 4, 5) if glob else (0, 1, 2)
                pk = p @ K
                var[iq][b, h, i] += scale ** 2 * (var_dD * pk ** 2 + u * u / 3.0 * ((dS ** 2) @ (K ** 2)))
                var[ik][b, h] += scale ** 2 * np.outer(var_dD * p ** 2 + u * u / 3.0 * dS ** 2, qi ** 2)
                var[iv][b, h] += u * u / 3.0 * np.outer(p ** 2, dO[i] ** 2)
    return [lam * np.sqrt(v) for v in var]


def compare_bound(name: str, got: np.ndarray, ref: np.ndarray, bound: np.ndarray, dtype: str,
                  factor: float = 2.0):
    """Assert |got - ref| <= factor * bound + u |ref| (+ a floor of 1e-6)
    elementwise where ref is defined; returns the largest ratio of the
    error to that allowance."""
    u = UNIT_ROUNDOFF[dtype]
    sel = ~np.isnan(ref)
    g, r, bd = got[sel], ref[sel], bound[sel]
    assert np.all(np.isfinite(g)), name + ": non-finite output"
    allow = factor * bd + u * np.abs(r) + 1e-6
    err = np.abs(g - r)
    worst = float((err / allow).max()) if err.size else 0.0
    k = int(np.argmax(err / allow)) if err.size else 0
    assert worst <= 1.0, "%s: error %.3e above its bound %.3e (ratio %.2f)" % (
        name, err[k], allow[k], worst)
    return worst
