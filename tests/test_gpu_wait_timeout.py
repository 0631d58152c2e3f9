"""Bounded device waits report DG_ETIMEOUT and leave the context usable.

Every wait of the library's kernels on a shared-memory barrier gives up after
a wall-time limit, records an error code and unwinds; the host reports it as
DG_ETIMEOUT at the next synchronising call.  The self-test makes one such wait
run out on purpose (a barrier nothing arrives on, with a limit of a few
milliseconds): no trap, no fault, the stream keeps working afterwards.
"""
import time

import pytest
import torch


@pytest.mark.gpu
def test_wait_that_runs_out_reports_timeout_and_recovers(dg):
    h = dg.dg_create(dict(vocab=8, canvas=4), None, dtype="fp32", max_batch=1, max_ctx=64)
    t0 = time.perf_counter()
    rc = dg.dg_selftest_wait_timeout(h, 5000)          # 5 ms
    dt = time.perf_counter() - t0
    assert rc == dg.DG_ETIMEOUT, dg.dg_last_error(h)
    assert "gave up" in dg.dg_last_error(h)
    assert dt < 5.0
    # the flag was cleared and the context works: a later call succeeds
    assert dg.dg_synchronize(h) == dg.DG_OK
    ctr = torch.arange(16, dtype=torch.int32, device="cuda").reshape(4, 4)
    key = torch.ones((4, 2), dtype=torch.int32, device="cuda")
    out = torch.zeros((4, 4), dtype=torch.int32, device="cuda")
    dg.dg_selftest_philox(h, ctr, key, out)
    dg.dg_synchronize(h)
    assert out.abs().sum().item() > 0
    # a second run times out again (the barrier state is per launch)
    assert dg.dg_selftest_wait_timeout(h, 1000) == dg.DG_ETIMEOUT
    assert dg.dg_selftest_wait_timeout(h, 0) == dg.DG_EINVAL          # limit out of range, nothing launched
    assert dg.dg_selftest_wait_timeout(h, 100001) == dg.DG_EINVAL
    h.close()
