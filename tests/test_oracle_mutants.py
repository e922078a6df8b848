"""Planted mistakes: each mutant of the oracle's C source must fail a pin.

The test copies oracle/lf_oracle.c, applies one plausible mistake (a dropped
term, a wrong sign or bound, a wrong index, a swapped projection), builds the
mutant into a temporary library, points the oracle wrapper at it and runs
the pins of test_oracle_pins.py.  At least one pin must fail for every
mutant; the real oracle passes all of them (test_oracle_pins.py).
CPU only.
"""
import ctypes
import os
import subprocess
import tempfile

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lf_oracle.c")

MUTANTS = {
    "window_off_by_one": ("if (k < -r || k > r) return 0;", "if (k < -r || k >= r) return 0;"),
    "causal_sign": ("if (causal && k > 0) return 0;", "if (causal && k < 0) return 0;"),
    "no_global_column": ("if (m[j] == 2) return 1;                /* every token sees global token */", ""),
    "dilation_ignored": ("if (dist % d != 0) return 0;", ""),
    "padding_keys_attended": ("if (m[i] == 0 || m[j] == 0) return 0;", "if (m[i] == 0) return 0;"),
    "scale_dropped": ("double s = scale * orc_dot(q, k + (size_t)j * hd, hd);\n        if (s > mx) mx = s;\n      }\n    if (mx == -INFINITY) { /* attends nothing",
                      "double s = orc_dot(q, k + (size_t)j * hd, hd);\n        if (s > mx) mx = s;\n      }\n    if (mx == -INFINITY) { /* attends nothing"),
    "global_row_local_proj": ("const double *v = glob ? vg : vs;\n    double mx = -INFINITY;\n    for (int j = 0; j < n; j++)\n      if (orc_bit(&A, i, j)) {\n        double s = scale * orc_dot(q, k + (size_t)j * hd, hd);\n        if (s > mx) mx = s;\n      }\n    if (mx == -INFINITY) { /* attends",
                              "const double *v = vs;\n    double mx = -INFINITY;\n    for (int j = 0; j < n; j++)\n      if (orc_bit(&A, i, j)) {\n        double s = scale * orc_dot(q, k + (size_t)j * hd, hd);\n        if (s > mx) mx = s;\n      }\n    if (mx == -INFINITY) { /* attends"),
    "bwd_delta_dropped": ("double ds = p * (orc_dot(g, vj, hd) - delta[i]);", "double ds = p * orc_dot(g, vj, hd);"),
    "bwd_dv_wrong_weight": ("dv[c] += p * g[c];", "dv[c] += ds * g[c];"),
    "bwd_dk_transposed": ("dk[c] += scale * ds * q[c];", "dk[c] += scale * ds * kj[c];"),
    "linear_weight_transposed": ("for (int k = 0; k < K; k++) s += xr[k] * wr[k];",
                                 "for (int k = 0; k < K; k++) s += xr[k] * w[(size_t)k * N + c];"),
    "linear_bias_dropped": ("y[(size_t)m * N + c] = s + (b ? b[c] : 0.0);", "y[(size_t)m * N + c] = s;"),
    "cross_mask_ignored": ("if (kmask && kmask[j] == 0) continue;\n      double s = scale",
                           "if (0) continue;\n      double s = scale"),
    "cross_unnormalised": ("for (int c = 0; c < hd; c++) oi[c] /= sum;", ""),
    "bwd_dq_unscaled": ("for (int c = 0; c < hd; c++) dq[c] += scale * ds * kj[c];",
                        "for (int c = 0; c < hd; c++) dq[c] += ds * kj[c];"),
}


def _pins():
    return [
        (pins.test_glossary_printed_pair_counts, ()),
        (pins.test_closed_form_counts_dilated_and_causal, (300, 17, 2)),
        *[(pins.test_pattern_brute_force_tiny, (s,)) for s in range(12)],
        (pins.test_global_symmetry_and_padding, ()),
        (pins.test_dense_special_case_w_ge_2n, ()),
        (pins.test_causal_dense_and_row0, ()),
        (pins.test_banded_matches_masked_dense, ()),
        (pins.test_global_row_is_dense_row_over_valid_keys, ()),
        (pins.test_dilation_split_invariant, (2,)),
        (pins.test_probability_rows, ()),
        (pins.test_backward_finite_differences, ("band_global_pad",)),
        (pins.test_backward_finite_differences, ("dilated",)),
        (pins.test_backward_zero_rows, ()),
        (pins.test_linear_matches_numpy_and_special_cases, ()),
        (pins.test_cross_attention_dense_numpy_and_global_row_equivalence, ()),
    ]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + name
    mutated = src.replace(old, new, 1)
    with tempfile.TemporaryDirectory() as tmp:
        c = os.path.join(tmp, "m.c")
        so = os.path.join(tmp, "m.so")
        open(c, "w").write(mutated)
        subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", so, c, "-lm"])
        real = oracle._load()
        lib = ctypes.CDLL(so)
        for f in ("threads", "pattern", "count_pairs", "probs_row", "fwd_head", "bwd_head", "linear",
                  "cross_head"):
            fn = getattr(lib, "lf_oracle_" + f)
            ref = getattr(real, "lf_oracle_" + f)
            fn.restype = ref.restype
            fn.argtypes = ref.argtypes
        monkeypatch.setattr(oracle, "_lib", lib)
        failed = []
        for fn, args in _pins():
            try:
                fn(*args)
            except (AssertionError, ValueError):
                failed.append(fn.__name__)
        assert failed, "mutant %s passed every pin" % name
