"""CPU checks of the measurement harness and the input generator: the bench's
reference arm (the oracle timed on the host cores) prints one well-formed
JSON line, and the synthetic workloads are deterministic, dtype-rounded and
shaped as declared."""
import json
import os
import subprocess
import sys

import numpy as np

from sparse_sliding_window_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True,
                         timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"].startswith("attended scores/s")
    assert d["unit"] == "scores/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "base_bf16"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_workloads_are_deterministic_and_rounded():
    wl = synth.WORKLOADS["base_bf16"]
    a = synth.make_inputs(wl, with_do=False)
    b = synth.make_inputs(wl, with_do=False)
    for k in ("qs", "ks", "vs", "qg", "kg", "vg", "mask"):
        assert np.array_equal(a[k], b[k]), k
    assert a["qs"].shape == (1, 12, 4096, 64) and a["qs"].dtype == np.uint16  # bf16 bit patterns
    # values are N(0, 0.5^2) rounded to bf16: re-rounding is the identity
    x = synth.as_float64(a["qs"], "bf16")
    assert np.array_equal(synth.round_to(x, "bf16"), a["qs"])
    assert abs(x.mean()) < 0.01 and abs(x.std() - 0.5) < 0.01
    # the QA question block: tokens 0..64 global, everything else local
    m = a["mask"][0]
    assert np.all(m[:65] == 2) and np.all(m[65:] == 1)


def test_batched_workload_structure():
    wl = synth.WORKLOADS["batched_f16"]
    m = synth.make_inputs(wl, with_do=False)["mask"]
    assert m.shape == (8, 4096)
    for b in range(8):
        L = int((m[b] != 0).sum())
        assert 2048 <= L <= 4096
        assert np.all(m[b, L:] == 0)  # padding tail
        g = np.flatnonzero(m[b] == 2)
        assert g[0] == 0 and len(g) == 17 and g.max() < L  # token 0 + 16 distinct in [1, L)


def test_algorithmic_bytes_of_base_workload():
    """The roofline denominator of the base workload, counted by hand: Q_s,
    K_s, V_s read and O written for 12 x 4096 rows of 128 bytes, Q_g at the
    65 global rows of each head, K_g and V_g in full, the int32 mask and the
    fp32 log-normaliser."""
    sys.path.insert(0, ROOT)
    import bench
    wl = synth.WORKLOADS["base_bf16"]
    mask = synth.make_inputs(wl, with_do=False)["mask"]
    rows = 12 * 4096
    expect = 4 * rows * 128 + 12 * 65 * 128 + 2 * rows * 128 + 4096 * 4 + rows * 4
    assert expect == 38061568
    assert bench.algorithmic_bytes(wl, mask) == expect


def test_algorithmic_bytes_of_charlm_workload():
    """Counted by hand: no global token, so K_g / V_g / Q_g are never read;
    8 heads x 23040 valid rows of 128 bytes for Q_s, K_s, V_s read and O
    written, the fp32 log-normaliser of every row and the int32 mask."""
    sys.path.insert(0, ROOT)
    import bench
    wl = synth.WORKLOADS["charlm_bf16"]
    mask = synth.make_inputs(wl, with_do=False)["mask"]
    rows = 8 * 23040
    expect = 4 * rows * 128 + rows * 4 + 23040 * 4
    assert expect == 95201280
    assert bench.algorithmic_bytes(wl, mask) == expect


def test_algorithmic_bytes_of_batched_workload():
    """Counted by hand from the seeded structure: the 8 sequences hold
    25229 valid tokens in all, each with 17 global tokens; per head, Q_s /
    K_s / V_s / K_g / V_g are read at the valid rows (every sequence has a
    global token), Q_g at the 136 global rows, O and the log-normaliser are
    written for all 8 x 4096 rows, and the mask is read once."""
    sys.path.insert(0, ROOT)
    import bench
    wl = synth.WORKLOADS["batched_f16"]
    mask = synth.make_inputs(wl, with_do=False)["mask"]
    assert int((mask != 0).sum()) == 25229 and int((mask == 2).sum()) == 136
    expect = (5 * 12 * 25229 * 128 + 12 * 136 * 128 + 12 * 8 * 4096 * 128 + 12 * 8 * 4096 * 4
              + 8 * 4096 * 4)
    assert expect == 246003200
    assert bench.algorithmic_bytes(wl, mask) == expect
