"""GPU: failure detection without a fault.

Extend's warps hand tiles to one another through shared-memory barriers, and
every wait on one is bounded in time.  Here a wait is made to run out on
purpose: the fault-injection hook of mg_set_extend_wait_limit withholds the
first score tile's hand-off (a barrier that nothing will complete), with the
bound shortened to 50 ms.  The kernel must give up, report
MG_ERR_DEVICE_TIMEOUT through mg_read_device_error, and leave the context
usable: the next normal call in the same process matches the oracle.  Nothing
traps, faults or hangs (the pages' engine bounds its own waits the same way,
"手写 mini-sglang 阶段一 · Engine 与采样器", §配置, distributed_timeout).
"""
import ctypes
import time

import pytest
import torch

from mg_testlib import GpuStep, assert_matches_oracle, oracle_extend
from paged_kv_attention_mg_b200 import mg
from paged_kv_attention_mg_b200 import workload as wl

pytestmark = pytest.mark.gpu


def _case():
    spec = wl.custom_spec("extend", [0, 300, 40], [200, 700, 41], 16, 8, 2000, seed=515)
    step = wl.make_step(spec)
    return step, wl.make_layer(step)


def test_extend_wait_that_runs_out_reports_a_timeout_and_the_context_survives():
    step, data = _case()
    g = GpuStep(step, data)
    g.store()
    assert mg.read_device_error() == 0
    lib = mg.load()
    try:
        mg.set_extend_wait_limit(50_000_000, inject_stall=True)  # 50 ms, one hand-off withheld
        t0 = time.perf_counter()
        g.extend()
        bits = ctypes.c_uint32(0)
        status = lib.mg_read_device_error(torch.cuda.current_stream().cuda_stream, ctypes.byref(bits))
        waited = time.perf_counter() - t0
    finally:
        mg.set_extend_wait_limit(0, inject_stall=False)  # the default bound, no injection
    assert status == 7, mg.STATUS.get(status, status)  # MG_ERR_DEVICE_TIMEOUT
    assert bits.value & mg.DEVERR_WAIT_TIMEOUT
    assert waited < 30.0  # the short bound applied, not the default one per CTA wave
    assert mg.read_device_error() == 0  # the word was cleared
    # the same process, the same context: a normal call is correct
    out = g.extend()
    assert mg.read_device_error() == 0
    assert_matches_oracle(out, oracle_extend(step, data), "extend after a timed-out launch")


def test_wait_limit_alone_changes_nothing():
    """A short bound with no injected stall: every wait is satisfied well within
    it, so the output is the oracle's and no error bit is set."""
    step, data = _case()
    g = GpuStep(step, data)
    g.store()
    try:
        mg.set_extend_wait_limit(200_000_000, inject_stall=False)
        out = g.extend()
        bits = mg.read_device_error()
    finally:
        mg.set_extend_wait_limit(0, inject_stall=False)
    assert bits == 0
    assert_matches_oracle(out, oracle_extend(step, data), "extend under a 200 ms wait bound")
