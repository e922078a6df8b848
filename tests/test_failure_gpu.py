"""Failure detection on the GPU without a fault: a bounded device wait that
runs out.

The tensor-core forward bounds every wait on an mbarrier.  The test hook
shortens the limit to 20 ms and makes CTA 0's producer leave one K/V tile
unloaded, so the MMA warp's wait for it expires: the kernel records
LF_ERR_DEVICE_TIMEOUT in the status word, lets the copies and MMAs it issued
finish, frees its tensor memory and returns.  Nothing faults, traps or hangs;
the next normal call on the same workspace must come back clean and match
the oracle.
"""
import numpy as np
import pytest

import oracle
from sparse_sliding_window_b200 import lf_attn as L
from sparse_sliding_window_b200 import synth
from tests import lfutil as U

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("skip", [1, 2])
def test_expired_wait_reports_timeout_then_recovers(skip):
    n, r = 640, 48
    m = np.ones((1, n), np.int32)
    m[0, [0, 300]] = 2
    wl = synth.custom("timeout", 1, 2, n, r, [1, 2], False, "bf16", m, seed=41)
    inp = synth.inputs_for(wl)
    g = U.gpu_inputs(inp, "bf16")
    att = L.LongformerAttention(1, 2, n, r, [1, 2], False, dtype="bf16", max_global=2,
                                kernel=L.LF_KERNEL_TC)
    try:
        L.lf_attn_set_test_hooks(20000, skip)
        att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    finally:
        L.lf_attn_set_test_hooks(0, 0)
    with pytest.raises(L.LfError) as e:
        att.status()
    assert e.value.code == L.LF_ERR_DEVICE_TIMEOUT
    # the context is usable and the next call is clean and correct
    o, lse = att.fwd(g["qs"], g["ks"], g["vs"], g["qg"], g["kg"], g["vg"], g["mask"])
    att.status()
    f = U.f64_inputs(inp, "bf16")
    ro, rl = oracle.fwd(r, [1, 2], False, U.scale_of(wl), m, f["qs"], f["ks"], f["vs"], f["qg"],
                        f["kg"], f["vg"])
    U.compare("after-timeout/o", U.to_f64(o), ro, "bf16")
    U.compare_lse(U.to_f64(lse), rl, "bf16")


def test_hook_argument_checks():
    with pytest.raises(L.LfError):
        L.lf_attn_set_test_hooks(0, -1)
    L.lf_attn_set_test_hooks(0, 0)
