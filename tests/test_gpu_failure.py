"""Failure detection on the GPU without a fault.

The pipeline kernel's waits are bounded by wall time.  A wait that nothing
completes must end with a status the host can read, and the context must
stay usable afterwards: the test runs the bounded-wait routine on an
mbarrier that nothing arrives at, reads the status, then runs a normal step
and checks it against the oracle.
"""
import time

import pytest
import torch

import zero_sharded_optimizer_reduce_b200 as Z
from test_gpu_step import Case, _adam

pytestmark = pytest.mark.gpu


def test_stuck_wait_reports_and_returns():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    Z.zero_test_wait_timeout(status, 200_000_000)        # 0.2 s
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == 2
    assert 0.15 <= elapsed < 5.0
    # the context is still usable: a normal step matches the oracle
    c = Case(8 * 300_007, 8, seed=500)
    c.run(_adam())
    ref, _, _ = c.expect(_adam())
    assert c.compare(ref) == [0, 0, 0, 0]


def test_zero_limit_gives_up_at_once():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Z.zero_test_wait_timeout(status, 0)
    torch.cuda.synchronize()
    assert int(status.item()) == 2
