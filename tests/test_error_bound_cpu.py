"""CPU checks of the derived error bound the large-score backward parity
test uses (tests/lfutil.py: bwd_error_bound, compare_bound): it admits the
rounding of the stored gradient, it is tight enough to catch a wrong sign,
and it does not swallow the reference (its norm stays well below it)."""
import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import synth
from tests import lfutil as U
from tests import test_parity_gpu as T


def _hot(name, dtype):
    c = T.CASES[name]
    wl = synth.custom(name, c["B"], c["H"], c["n"], c["r"], c["dil"], c["causal"], dtype, c["mask"],
                      seed=11, in_scale=c["in_scale"], backward=True)
    inp = synth.inputs_for(wl)
    for k in ("vs", "vg"):
        inp[k] = synth.round_to(synth.as_float64(inp[k], dtype) / c["in_scale"], dtype)
    f = U.f64_inputs(inp, dtype)
    scale = U.scale_of(wl)
    ref = oracle.bwd(c["r"], c["dil"], c["causal"], scale, inp["mask"], f["qs"], f["ks"], f["vs"],
                     f["qg"], f["kg"], f["vg"], f["do"])
    return ref, U.bwd_error_bound(c, scale, inp["mask"], f, dtype)


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_bound_admits_rounding_and_rejects_sign_flip(dtype):
    ref, bound = _hot("hot_scores", dtype)
    for k in range(6):
        r = ref[k]
        rounded = synth.as_float64(synth.round_to(r, dtype), dtype)
        U.compare_bound("rounded", rounded, r, bound[k], dtype, factor=1.0)
        # the element whose magnitude most exceeds its allowance, negated
        margin = np.abs(r) / (bound[k] + U.UNIT_ROUNDOFF[dtype] * np.abs(r) + 1e-6)
        idx = np.unravel_index(np.nanargmax(margin), r.shape)
        bad = r.copy()
        bad[idx] = -bad[idx]
        with pytest.raises(AssertionError):
            U.compare_bound("flipped", bad, r, bound[k], dtype, factor=1.0)


def test_bound_not_vacuous():
    ref, bound = _hot("hot_scores", "bf16")
    for k in range(6):
        sel = ~np.isnan(ref[k])
        assert np.linalg.norm(bound[k][sel]) < 0.25 * np.linalg.norm(ref[k][sel]), k
