"""CPU oracle for Longformer self-attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``sparse_sliding_window_b200``) never imports it, and the two
share no code: this package wraps ``lf_oracle.c`` (plain C, double precision,
OpenMP over rows) through ctypes.

What it computes is documented in ``lf_oracle.c``: the attention pattern of
each head is materialised as an explicit n x n bit matrix from the literal
per-pair rule, then softmax attention is evaluated in float64 over its set
bits.  Inputs are the generator's values AFTER rounding to the run's dtype,
upcast to float64, so the tolerance measures the kernels and not the input
quantisation.

Every function of the oracle is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` against facts the pages and the mathematics fix
(the printed pair counts of the ultralytics glossary example, closed-form
counts, brute-force enumeration, dense attention as a special case, the
dilation split invariant, the causal row-0 case, row sums, symmetry of the
global pattern and central finite differences for the backward).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lf_oracle.c")
_LIB = os.path.join(_HERE, "liblf_oracle.so")
_lib = None

ERRORS = {1: "invalid argument", 2: "out of memory", 3: "unsupported (causal with global tokens)"}


def build(force: bool = False) -> str:
    """Compile lf_oracle.c into liblf_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i32, dbl, p = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.lf_oracle_threads.restype = i32
        lib.lf_oracle_pattern.argtypes = [i32, i32, i32, i32, p, p]
        lib.lf_oracle_count_pairs.argtypes = [i32, i32, i32, i32, p, p]
        lib.lf_oracle_probs_row.argtypes = [i32, i32, i32, i32, i32, dbl, p, p, p, p, p, i32, p]
        lib.lf_oracle_fwd_head.argtypes = [i32, i32, i32, i32, i32, dbl, p] + [p] * 6 + [p, p]
        lib.lf_oracle_bwd_head.argtypes = [i32, i32, i32, i32, i32, dbl, p] + [p] * 7 + [p] * 6
        lib.lf_oracle_linear.argtypes = [i32, i32, i32, p, p, p, p]
        lib.lf_oracle_cross_head.argtypes = [i32, i32, i32, dbl, p, p, p, p, p, p]
        for f in ("pattern", "count_pairs", "probs_row", "fwd_head", "bwd_head", "linear", "cross_head"):
            getattr(lib, "lf_oracle_" + f).restype = i32
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(st: int):
    if st != 0:
        raise ValueError("oracle: " + ERRORS.get(st, "error %d" % st))


def _mask(m) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(m, dtype=np.int32))


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def threads() -> int:
    """OpenMP threads the oracle uses (the cores of the CPU baseline)."""
    return int(_load().lf_oracle_threads())


def pattern(n: int, r: int, d: int, causal: bool, mask) -> np.ndarray:
    """The materialised attention pattern A of one head: uint8 [n, n]."""
    m = _mask(mask)
    assert m.shape == (n,)
    out = np.zeros((n, n), dtype=np.uint8)
    _check(_load().lf_oracle_pattern(n, r, d, int(causal), _ptr(m), _ptr(out)))
    return out


def count_pairs(n: int, r: int, d: int, causal: bool, mask) -> int:
    """popcount(A): attended (query, key) pairs of one head."""
    m = _mask(mask)
    assert m.shape == (n,)
    c = np.zeros(1, dtype=np.int64)
    _check(_load().lf_oracle_count_pairs(n, r, d, int(causal), _ptr(m), _ptr(c)))
    return int(c[0])


def probs_row(i: int, r: int, d: int, causal: bool, scale: float, mask, qs, ks, qg, kg) -> np.ndarray:
    """Row i of the attention probabilities of one head (float64 [n])."""
    m = _mask(mask)
    qs, ks, qg, kg = map(_f64, (qs, ks, qg, kg))
    n, hd = qs.shape
    out = np.zeros(n, dtype=np.float64)
    _check(_load().lf_oracle_probs_row(n, hd, r, d, int(causal), float(scale), _ptr(m),
                                       _ptr(qs), _ptr(ks), _ptr(qg), _ptr(kg), int(i), _ptr(out)))
    return out


def fwd_head(r: int, d: int, causal: bool, scale: float, mask, qs, ks, vs, qg, kg, vg):
    """Forward of one head: returns (o float64 [n, hd], lse float64 [n])."""
    m = _mask(mask)
    t = [_f64(x) for x in (qs, ks, vs, qg, kg, vg)]
    n, hd = t[0].shape
    for x in t:
        assert x.shape == (n, hd)
    o = np.zeros((n, hd), dtype=np.float64)
    lse = np.zeros(n, dtype=np.float64)
    _check(_load().lf_oracle_fwd_head(n, hd, r, d, int(causal), float(scale), _ptr(m),
                                      *[_ptr(x) for x in t], _ptr(o), _ptr(lse)))
    return o, lse


def bwd_head(r: int, d: int, causal: bool, scale: float, mask, qs, ks, vs, qg, kg, vg, dO):
    """Backward of one head for L = sum(o * dO).

    Returns (dqs, dks, dvs, dqg, dkg, dvg), each float64 [n, hd].
    """
    m = _mask(mask)
    t = [_f64(x) for x in (qs, ks, vs, qg, kg, vg, dO)]
    n, hd = t[0].shape
    outs = [np.zeros((n, hd), dtype=np.float64) for _ in range(6)]
    _check(_load().lf_oracle_bwd_head(n, hd, r, d, int(causal), float(scale), _ptr(m),
                                      *[_ptr(x) for x in t], *[_ptr(x) for x in outs]))
    return tuple(outs)


def fwd(r: int, dilation, causal: bool, scale: float, mask, qs, ks, vs, qg, kg, vg, heads=None):
    """Forward over [B, H, n, hd] float64 arrays; ``heads`` = optional list of
    (b, h) to evaluate (the others are left as NaN).  ``dilation`` is [H]."""
    B, H, n, hd = np.shape(qs)
    o = np.full((B, H, n, hd), np.nan)
    lse = np.full((B, H, n), np.nan)
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in sel:
        o[b, h], lse[b, h] = fwd_head(r, int(dilation[h]), causal, scale, mask[b],
                                      qs[b, h], ks[b, h], vs[b, h], qg[b, h], kg[b, h], vg[b, h])
    return o, lse


def bwd(r: int, dilation, causal: bool, scale: float, mask, qs, ks, vs, qg, kg, vg, dO, heads=None):
    """Backward over [B, H, n, hd] arrays; returns six gradients (NaN outside ``heads``)."""
    B, H, n, hd = np.shape(qs)
    outs = [np.full((B, H, n, hd), np.nan) for _ in range(6)]
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in sel:
        gs = bwd_head(r, int(dilation[h]), causal, scale, mask[b], qs[b, h], ks[b, h], vs[b, h],
                      qg[b, h], kg[b, h], vg[b, h], dO[b, h])
        for k in range(6):
            outs[k][b, h] = gs[k]
    return tuple(outs)


def counts(r: int, dilation, causal: bool, mask, H: int) -> np.ndarray:
    """Attended pairs per (b, h): int64 [B, H]."""
    B, n = np.shape(mask)
    out = np.zeros((B, H), dtype=np.int64)
    cache = {}
    for b in range(B):
        for h in range(H):
            key = (b, int(dilation[h]))
            if key not in cache:
                cache[key] = count_pairs(n, r, int(dilation[h]), causal, mask[b])
            out[b, h] = cache[key]
    return out


def linear(x, w, b=None) -> np.ndarray:
    """The affine map y = x w^T + b over the last axis of x (float64), with
    w in the [out_features, in_features] layout: the projections into
    Qs/Ks/Vs/Qg/Kg/Vg and the output projection around the attention."""
    x = _f64(x)
    w = _f64(w)
    N, K = w.shape
    assert x.shape[-1] == K
    lead = x.shape[:-1]
    M = int(np.prod(lead)) if lead else 1
    xb = np.ascontiguousarray(x.reshape(M, K))
    bb = None if b is None else _f64(b)
    assert bb is None or bb.shape == (N,)
    y = np.zeros((M, N), dtype=np.float64)
    _check(_load().lf_oracle_linear(M, N, K, _ptr(xb), _ptr(w), None if bb is None else _ptr(bb), _ptr(y)))
    return y.reshape(lead + (N,))


def cross_head(scale: float, kmask, q, k, v):
    """Cross-attention of one head: q [Lq, hd] against k, v [Lk, hd], keys
    with kmask != 0 (kmask None: every key).  Returns (o [Lq, hd], lse [Lq])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Lq, hd = q.shape
    Lk = k.shape[0]
    assert k.shape == (Lk, hd) and v.shape == (Lk, hd)
    m = None if kmask is None else _mask(kmask)
    assert m is None or m.shape == (Lk,)
    o = np.zeros((Lq, hd), dtype=np.float64)
    lse = np.zeros(Lq, dtype=np.float64)
    _check(_load().lf_oracle_cross_head(Lq, Lk, hd, float(scale), None if m is None else _ptr(m),
                                        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse)))
    return o, lse


def cross(scale: float, kmask, q, k, v, heads=None):
    """Cross-attention over q [B, H, Lq, hd] and k, v [B, H, Lk, hd] with a
    key mask [B, Lk] (or None); ``heads`` = optional list of (b, h) to
    evaluate (the others are left as NaN).  Returns (o, lse)."""
    B, H, Lq, hd = np.shape(q)
    o = np.full((B, H, Lq, hd), np.nan)
    lse = np.full((B, H, Lq), np.nan)
    sel = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in sel:
        o[b, h], lse[b, h] = cross_head(scale, None if kmask is None else kmask[b], q[b, h], k[b, h],
                                        v[b, h])
    return o, lse

