"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself:
  * the pair counts printed by the glossary pages' worked example,
  * closed-form pair counts of the band (non-causal, causal, dilated),
  * brute-force enumeration of the pattern on tiny inputs,
  * dense softmax attention (numpy matmul + exp) as the w >= 2n special case,
  * a dense attention row with Qg/Kg/Vg for global rows,
  * the dilation split invariant, the causal row-0 case, causal dense,
  * probability rows (sum 1, support == pattern), global symmetry,
  * central finite differences of the forward for the backward.
No GPU is needed (marker: not gpu).
"""
import math
import os

import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "glossary_pair_counts.txt")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _dense_attention(q, k, v, scale, allowed):
    """Plain dense softmax attention in float64 (numpy), rows with no allowed
    key give 0 / -inf."""
    s = scale * (q @ k.T)
    s = np.where(allowed, s, -np.inf)
    mx = s.max(axis=1, keepdims=True)
    o = np.zeros_like(q)
    lse = np.full(q.shape[0], -np.inf)
    ok = np.isfinite(mx[:, 0])
    e = np.exp(s[ok] - mx[ok])
    o[ok] = (e @ v) / e.sum(axis=1, keepdims=True)
    lse[ok] = mx[ok, 0] + np.log(e.sum(axis=1))
    return o, lse


# ------------------------------------------------------------------ counts --

def test_glossary_printed_pair_counts():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for n_s, full_s, lf_s in rows:
        n = int(n_s)
        m = np.ones(n, np.int32)
        m[0] = 2
        c = oracle.count_pairs(n, 256, 1, False, m)
        assert "%.1f" % (c / 1e6) == lf_s
        full = oracle.count_pairs(n, n, 1, False, np.ones(n, np.int32))
        assert "%.1f" % (full / 1e6) == full_s
        assert full == n * n


@pytest.mark.parametrize("n", [1024, 2048, 4096])
def test_closed_form_band_plus_global0(n):
    r = 256
    m = np.ones(n, np.int32)
    m[0] = 2
    band = n * (2 * r + 1) - r * (r + 1)
    expect = band + 2 * (n - r - 1)   # token 0's row and column beyond its window
    assert oracle.count_pairs(n, r, 1, False, m) == expect
    assert expect == {1024: 461054, 2048: 988414, 4096: 2043134}[n]


@pytest.mark.parametrize("n,r,d", [(300, 17, 1), (300, 17, 2), (301, 9, 3), (64, 5, 4)])
def test_closed_form_counts_dilated_and_causal(n, r, d):
    m = np.ones(n, np.int32)
    # each residue class rho of length n_rho >= r is an undilated band
    assert oracle.count_pairs(n, r, d, False, m) == n * (2 * r + 1) - d * r * (r + 1)
    assert oracle.count_pairs(n, r, d, True, m) == n * (r + 1) - d * r * (r + 1) // 2


def _brute_sets(n, r, d, causal, m):
    """Enumerate each row's key set constructively (window steps k*d, then the
    global tokens), independent of the oracle's per-pair predicate."""
    A = np.zeros((n, n), np.uint8)
    glob = [g for g in range(n) if m[g] == 2]
    for i in range(n):
        if m[i] == 0:
            continue
        if m[i] == 2:
            keys = {j for j in range(n) if m[j] != 0}
        else:
            hi = 0 if causal else r
            keys = {i + k * d for k in range(-r, hi + 1)}
            keys = {j for j in keys if 0 <= j < n and m[j] != 0}
            keys |= set(glob)
        for j in keys:
            A[i, j] = 1
    return A


@pytest.mark.parametrize("seed", range(12))
def test_pattern_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    r = int(rng.integers(0, 7))
    d = int(rng.integers(1, 4))
    causal = bool(seed % 3 == 0)
    m = rng.choice([0, 1, 1, 1, 2], size=n).astype(np.int32)
    if causal:
        m[m == 2] = 1
    A = oracle.pattern(n, r, d, causal, m)
    assert np.array_equal(A, _brute_sets(n, r, d, causal, m))
    assert oracle.count_pairs(n, r, d, causal, m) == int(A.sum())


def test_global_symmetry_and_padding():
    n, r = 50, 3
    m = np.ones(n, np.int32)
    m[[0, 7, 31]] = 2
    m[40:] = 0
    A = oracle.pattern(n, r, 2, False, m)
    valid = m != 0
    for g in (0, 7, 31):
        assert A[g, valid].all() and A[valid, g].all()
    assert not A[~valid, :].any() and not A[:, ~valid].any()


def test_causal_with_global_rejected():
    m = np.ones(10, np.int32)
    m[0] = 2
    with pytest.raises(ValueError):
        oracle.count_pairs(10, 2, 1, True, m)


# ----------------------------------------------------------------- forward --

def test_dense_special_case_w_ge_2n():
    n, hd = 96, 64
    q, k, v = (_rand((n, hd), s) for s in (1, 2, 3))
    m = np.ones(n, np.int32)
    scale = 1 / math.sqrt(hd)
    o, lse = oracle.fwd_head(n, 1, False, scale, m, q, k, v, q * 0, k * 0, v * 0)
    o2, lse2 = _dense_attention(q, k, v, scale, np.ones((n, n), bool))
    assert np.max(np.abs(o - o2)) < 1e-12
    assert np.max(np.abs(lse - lse2)) < 1e-12


def test_causal_dense_and_row0():
    n, hd = 80, 64
    q, k, v = (_rand((n, hd), s) for s in (4, 5, 6))
    m = np.ones(n, np.int32)
    scale = 0.125
    o, lse = oracle.fwd_head(n, 1, True, scale, m, q, k, v, q, k, v)
    o2, _ = _dense_attention(q, k, v, scale, np.tril(np.ones((n, n), bool)))
    assert np.max(np.abs(o - o2)) < 1e-12
    o3, _ = oracle.fwd_head(7, 1, True, scale, m, q, k, v, q, k, v)
    assert np.array_equal(o3[0], v[0])


def test_banded_matches_masked_dense():
    """Band + padding + globals equals dense attention restricted to the
    brute-force pattern, with Qg/Kg/Vg on global rows."""
    n, hd, r = 70, 16, 5
    m = np.ones(n, np.int32)
    m[[3, 50]] = 2
    m[66:] = 0
    qs, ks, vs, qg, kg, vg = (_rand((n, hd), 10 + s) for s in range(6))
    scale = 0.3
    A = _brute_sets(n, r, 1, False, m).astype(bool)
    o, lse = oracle.fwd_head(r, 1, False, scale, m, qs, ks, vs, qg, kg, vg)
    ol, lsel = _dense_attention(qs, ks, vs, scale, A)
    og, lseg = _dense_attention(qg, kg, vg, scale, A)
    isg = m == 2
    assert np.max(np.abs(o[~isg] - ol[~isg])) < 1e-12
    assert np.max(np.abs(o[isg] - og[isg])) < 1e-12
    assert np.array_equal(np.isinf(lse), m == 0)
    assert np.all(o[m == 0] == 0)


def test_global_row_is_dense_row_over_valid_keys():
    n, hd = 120, 64
    m = np.ones(n, np.int32)
    m[0] = 2
    m[100:] = 0
    t = [_rand((n, hd), 20 + s) for s in range(6)]
    o, lse = oracle.fwd_head(8, 1, False, 0.125, m, *t)
    valid = (m != 0)[None, :]
    og, lseg = _dense_attention(t[3][:1], t[4], t[5], 0.125, valid)
    assert np.max(np.abs(o[0] - og[0])) < 1e-12
    assert abs(lse[0] - lseg[0]) < 1e-12


@pytest.mark.parametrize("d", [2, 3])
def test_dilation_split_invariant(d):
    n, hd, r = 61, 8, 4
    m = np.ones(n, np.int32)
    t = [_rand((n, hd), 40 + s) for s in range(6)]
    o, lse = oracle.fwd_head(r, d, False, 0.5, m, *t)
    for rho in range(d):
        idx = np.arange(rho, n, d)
        sub = [x[idx] for x in t]
        os_, lses = oracle.fwd_head(r, 1, False, 0.5, m[idx], *sub)
        assert np.max(np.abs(o[idx] - os_)) < 1e-13
        assert np.max(np.abs(lse[idx] - lses)) < 1e-13


def test_probability_rows():
    n, hd, r = 90, 16, 6
    m = np.ones(n, np.int32)
    m[[0, 45]] = 2
    m[80:] = 0
    qs, ks, vs, qg, kg, vg = (_rand((n, hd), 60 + s) for s in range(6))
    A = oracle.pattern(n, r, 2, False, m)
    o, _ = oracle.fwd_head(r, 2, False, 0.25, m, qs, ks, vs, qg, kg, vg)
    for i in (0, 1, 2, 44, 45, 46, 79, 85):
        p = oracle.probs_row(i, r, 2, False, 0.25, m, qs, ks, qg, kg)
        if m[i] == 0:
            assert not p.any()
            continue
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p >= 0)
        assert np.array_equal(p > 0, A[i] == 1)
        v = vg if m[i] == 2 else vs
        assert np.max(np.abs(p @ v - o[i])) < 1e-12


# ---------------------------------------------------------------- backward --

@pytest.mark.parametrize("case", ["band_global_pad", "dilated", "causal"])
def test_backward_finite_differences(case):
    n, hd = 14, 4
    m = np.ones(n, np.int32)
    r, d, causal = 2, 1, False
    if case == "band_global_pad":
        m[[1, 9]] = 2
        m[12:] = 0
    elif case == "dilated":
        d = 2
        m[5] = 2
    else:
        causal = True
        d = 2
    t = [_rand((n, hd), 80 + s) for s in range(6)]
    dO = _rand((n, hd), 99)
    scale = 0.7
    grads = oracle.bwd_head(r, d, causal, scale, m, *t, dO)

    def loss(tt):
        o, _ = oracle.fwd_head(r, d, causal, scale, m, *tt)
        return float(np.sum(o * dO))

    h = 1e-6
    for which in range(6):
        num = np.zeros((n, hd))
        for idx in np.ndindex(n, hd):
            tp = [x.copy() for x in t]
            tm = [x.copy() for x in t]
            tp[which][idx] += h
            tm[which][idx] -= h
            num[idx] = (loss(tp) - loss(tm)) / (2 * h)
        err = np.max(np.abs(num - grads[which])) / max(1.0, np.max(np.abs(num)))
        assert err < 1e-6, (case, which, err)


def test_backward_zero_rows():
    n, hd = 20, 4
    m = np.ones(n, np.int32)
    m[15:] = 0
    m[2] = 2
    t = [_rand((n, hd), 120 + s) for s in range(6)]
    g = oracle.bwd_head(3, 1, False, 0.5, m, *t, _rand((n, hd), 130))
    dqs, dks, dvs, dqg, dkg, dvg = g
    assert not dqs[15:].any() and not dks[15:].any() and not dvs[15:].any()
    assert not dkg[15:].any() and not dvg[15:].any()
    assert not dqs[2].any()                     # global row: gradient goes to Qg
    assert not np.delete(dqg, 2, axis=0).any()  # only the global row has dQg


# --------------------------------------------------------------- generator --

def test_generator_is_counter_based_and_normal():
    a = synth.normals(7, 1, 1000)
    b = synth.normals(7, 1, 1 << 23)[:1000]
    assert np.array_equal(a, b)
    x = synth.normals(7, 2, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    bf = synth.round_to(np.array([1.0, 1.00390625, 1.005859375, -2.5]), "bf16")
    assert list(synth.as_float64(bf, "bf16")) == [1.0, 1.0, 1.0078125, -2.5]


def test_workload_masks():
    for name, wl in synth.WORKLOADS.items():
        m = synth.build_mask(wl)
        assert m.shape == (wl.B, wl.n)
        assert set(np.unique(m)) <= {0, 1, 2}
    m = synth.build_mask(synth.WORKLOADS["batched_f16"])
    for b in range(8):
        L = int((m[b] != 0).sum())
        assert 2048 <= L <= 4096 and (m[b, L:] == 0).all()
        assert m[b, 0] == 2 and int((m[b] == 2).sum()) == 17
    m = synth.build_mask(synth.WORKLOADS["base_bf16"])
    assert (m[0, :65] == 2).all() and (m[0, 65:] == 1).all()


# ---------------------------------------------------------------- projections

def test_linear_matches_numpy_and_special_cases():
    """oracle.linear (the projections either side of the attention) against
    numpy's matmul on non-square, non-symmetric shapes, and against what the
    definition fixes: an identity weight copies x, a zero input gives the
    bias, and the map is linear in x without the bias."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 5, 6))
    w = rng.standard_normal((4, 6))
    b = rng.standard_normal(4)
    np.testing.assert_allclose(oracle.linear(x, w, b), x @ w.T + b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(oracle.linear(x, w), x @ w.T, rtol=0, atol=1e-12)
    sq = rng.standard_normal((6, 6))  # square, non-symmetric: a transposed index shows
    np.testing.assert_allclose(oracle.linear(x, sq), x @ sq.T, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(oracle.linear(x, np.eye(6)), x)
    np.testing.assert_array_equal(oracle.linear(np.zeros((2, 6)), w, b), np.tile(b, (2, 1)))
    x2 = rng.standard_normal((3, 5, 6))
    np.testing.assert_allclose(oracle.linear(2.5 * x + x2, w), 2.5 * oracle.linear(x, w) + oracle.linear(x2, w),
                               rtol=0, atol=1e-12)


# ------------------------------------------------------------ cross-attention

def test_cross_attention_dense_numpy_and_global_row_equivalence():
    """oracle.cross_head (LED decoder cross-attention) against a dense numpy
    softmax attention over the valid keys, and against the oracle's own
    self-attention where they coincide: a global query row attends every
    valid key with the global projections, so its output equals cross-
    attention of that query over K_g, V_g with the mask as the key mask."""
    rng = np.random.default_rng(11)
    Lq, Lk, hd, scale = 7, 40, 16, 0.25
    q, k, v = (rng.standard_normal((L, hd)) for L in (Lq, Lk, Lk))
    km = np.ones(Lk, np.int32)
    km[[3, 17, 39]] = 0
    o, lse = oracle.cross_head(scale, km, q, k, v)
    s = scale * q @ k.T
    s[:, km == 0] = -np.inf
    mx = s.max(axis=1, keepdims=True)
    p = np.exp(s - mx)
    np.testing.assert_allclose(o, (p / p.sum(axis=1, keepdims=True)) @ v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, mx[:, 0] + np.log(p.sum(axis=1)), rtol=0, atol=1e-12)
    # no key mask = every key
    o2, _ = oracle.cross_head(scale, None, q, k, v)
    s2 = scale * q @ k.T
    p2 = np.exp(s2 - s2.max(axis=1, keepdims=True))
    np.testing.assert_allclose(o2, (p2 / p2.sum(axis=1, keepdims=True)) @ v, rtol=0, atol=1e-12)
    # every key masked: o = 0, lse = -inf
    o3, lse3 = oracle.cross_head(scale, np.zeros(Lk, np.int32), q, k, v)
    assert np.all(o3 == 0) and np.all(np.isneginf(lse3))
    # the global-row special case of the self-attention oracle
    n = 50
    mask = np.ones(n, np.int32)
    mask[[0, 21]] = 2
    mask[45:] = 0
    t = {nm: rng.standard_normal((n, hd)) for nm in ("qs", "ks", "vs", "qg", "kg", "vg")}
    fo, flse = oracle.fwd_head(4, 1, False, scale, mask, t["qs"], t["ks"], t["vs"], t["qg"], t["kg"], t["vg"])
    co, clse = oracle.cross_head(scale, (mask != 0).astype(np.int32), t["qg"][[0, 21]], t["kg"], t["vg"])
    np.testing.assert_allclose(co, fo[[0, 21]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(clse, flse[[0, 21]], rtol=0, atol=1e-12)
    # permuting the keys with their values leaves every output unchanged
    perm = rng.permutation(Lk)
    o4, lse4 = oracle.cross_head(scale, km[perm], q, k[perm], v[perm])
    np.testing.assert_allclose(o4, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse4, lse, rtol=0, atol=1e-12)
