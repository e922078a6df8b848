"""Pins of the oracle's batched wrappers ``oracle.fwd``, ``oracle.bwd`` and
``oracle.counts`` (CPU only).

The wrappers pick the dilation of each head, the mask of each sequence and
the (b, h) slices of the inputs, and cache pair counts per (b, d).  A slip
there (every head given head 0's dilation, sequence 0's mask everywhere, a
cache key that forgets b) would pass the single-head pins and fail only
against the GPU, where a matching kernel bug could hide it.  So the wrappers
are checked here on B = 2 sequences with different masks and per-head
dilations [1, 2, 3]:
  * against explicit single-head calls with each head's own d and mask;
  * against the dilation split of the pages' dilated window ("gaps of size
    d", segmentfault page, section 扩张滑动窗口): on a sequence without
    global tokens, a head with dilation d is d independent undilated bands,
    one per residue sub-sequence rho, rho + d, ...; its outputs and
    gradients equal the d = 1 results of those sub-sequences re-interleaved,
    and its pair count is their sum.  This check never passes d to the
    oracle, so it does not lean on the function under test.
Planted mutants of the wrapper source must fail the same check.
"""
import inspect
import math

import numpy as np
import pytest

import oracle

B, H, n, R = 2, 3, 61, 4
DIL = [1, 2, 3]
SCALE = 1.0 / math.sqrt(8)


def _inputs():
    rng = np.random.default_rng(404)
    t = {k: rng.standard_normal((B, H, n, 8)) for k in ("qs", "ks", "vs", "qg", "kg", "vg", "do")}
    m = np.ones((B, n), np.int32)
    m[0, [0, 17, 40]] = 2      # sequence 0: global tokens
    m[1, 50:] = 0              # sequence 1: padding tail, no global token
    m[1, 9] = 0                # and a hole inside
    return t, m


def _split_fwd(t, m, b, h, d):
    """Head (b, h) with dilation d from d undilated sub-sequence calls."""
    o = np.zeros((n, 8))
    lse = np.zeros(n)
    for rho in range(d):
        sl = slice(rho, None, d)
        o[sl], lse[sl] = oracle.fwd_head(R, 1, False, SCALE, m[b, sl], *[t[k][b, h, sl] for k in
                                         ("qs", "ks", "vs", "qg", "kg", "vg")])
    return o, lse


def _split_bwd(t, m, b, h, d):
    g = [np.zeros((n, 8)) for _ in range(6)]
    for rho in range(d):
        sl = slice(rho, None, d)
        part = oracle.bwd_head(R, 1, False, SCALE, m[b, sl], *[t[k][b, h, sl] for k in
                               ("qs", "ks", "vs", "qg", "kg", "vg", "do")])
        for k in range(6):
            g[k][sl] = part[k]
    return g


def check_wrappers(fwd, bwd, counts):
    """Raises AssertionError when a wrapper disagrees with the pins."""
    t, m = _inputs()
    args = [t[k] for k in ("qs", "ks", "vs", "qg", "kg", "vg")]
    o, lse = fwd(R, DIL, False, SCALE, m, *args)
    grads = bwd(R, DIL, False, SCALE, m, *args, t["do"])
    cnt = counts(R, DIL, False, m, H)
    assert cnt.shape == (B, H)
    for b in range(B):
        for h in range(H):
            d = DIL[h]
            ro, rl = oracle.fwd_head(R, d, False, SCALE, m[b], *[a[b, h] for a in args])
            np.testing.assert_allclose(o[b, h], ro, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], rl, rtol=0, atol=1e-12)
            rg = oracle.bwd_head(R, d, False, SCALE, m[b], *[a[b, h] for a in args], t["do"][b, h])
            for k in range(6):
                np.testing.assert_allclose(grads[k][b, h], rg[k], rtol=0, atol=1e-12)
            assert cnt[b, h] == oracle.count_pairs(n, R, d, False, m[b])
    # sequence 1 has no global token: the dilation split holds there
    b = 1
    for h in range(H):
        d = DIL[h]
        so, sl = _split_fwd(t, m, b, h, d)
        np.testing.assert_allclose(o[b, h], so, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b, h], sl, rtol=0, atol=1e-12)
        sg = _split_bwd(t, m, b, h, d)
        for k in range(6):
            np.testing.assert_allclose(grads[k][b, h], sg[k], rtol=0, atol=1e-12)
        split_count = sum(oracle.count_pairs(len(m[b, rho::d]), R, 1, False, m[b, rho::d])
                          for rho in range(d))
        assert cnt[b, h] == split_count


def test_wrappers_match_single_head_calls_and_dilation_split():
    check_wrappers(oracle.fwd, oracle.bwd, oracle.counts)


# (wrapper, source text, mutated text): plausible slips in the per-head dispatch
MUTANTS = {
    "fwd_dilation_of_head0": ("fwd", "int(dilation[h])", "int(dilation[0])"),
    "fwd_mask_of_seq0": ("fwd", "mask[b],", "mask[0],"),
    "bwd_dilation_of_head0": ("bwd", "int(dilation[h])", "int(dilation[0])"),
    "bwd_dO_of_head0": ("bwd", "dO[b, h]", "dO[b, 0]"),
    "counts_cache_ignores_b": ("counts", "key = (b, int(dilation[h]))", "key = (0, int(dilation[h]))"),
    "counts_dilation_of_head0": ("counts", "count_pairs(n, r, int(dilation[h])",
                                 "count_pairs(n, r, int(dilation[0])"),
}


def _mutant(fn_name, old, new):
    src = inspect.getsource(getattr(oracle, fn_name))
    assert src.count(old) >= 1, (fn_name, old)
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant %s>" % fn_name, "exec"), ns)
    return ns[fn_name]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_wrapper_mutant_is_caught(name):
    fn_name, old, new = MUTANTS[name]
    fns = {"fwd": oracle.fwd, "bwd": oracle.bwd, "counts": oracle.counts}
    fns[fn_name] = _mutant(fn_name, old, new)
    with pytest.raises(AssertionError):
        check_wrappers(fns["fwd"], fns["bwd"], fns["counts"])
