"""The device timeout path: a bounded wait that runs out is reported, not hung.

Every wait in the library's kernels (mbarriers, grid barriers) gives up after a
limit of %globaltimer and records a timeout in the device status word instead
of spinning for ever.  bl_selftest_wait_timeout runs that same bounded wait on
an mbarrier phase that nothing completes, with a limit of milliseconds; the
status must come back as BL_ERR_DEVICE_TIMEOUT once, be cleared by reading it,
and leave the context usable."""
import time

import numpy as np
import pytest

import oracle
from workloads import random_problem

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_is_reported(bl):
    import torch
    assert bl.sync_status() == "BL_OK"
    t0 = time.perf_counter()
    bl.selftest_wait_timeout(2_000_000)          # 2 ms
    assert bl.sync_status() == "BL_ERR_DEVICE_TIMEOUT"
    assert time.perf_counter() - t0 < 5.0
    assert bl.sync_status() == "BL_OK"           # read and cleared
    # the context still computes
    p = random_problem(11, 2, 640, 96)
    Wd, beta = bl.quantize_weights_pack5(torch.from_numpy(p.W).cuda(), p.eps)
    Y = bl.linear(torch.from_numpy(np.ascontiguousarray(p.X)).cuda(), Wd, bl.PACK5, p.N, p.K, beta, eps=p.eps)
    assert bl.sync_status() == "BL_OK"
    ref = oracle.bitlinear(p.X, p.W, p.eps)["Y"]
    np.testing.assert_allclose(Y.cpu().numpy(), ref, rtol=0, atol=0)


def test_timeout_limits_are_checked(bl):
    for limit in (0, 999, 10 ** 9 + 1):
        with pytest.raises(bl.BitLinearError):
            bl.selftest_wait_timeout(limit)
    assert bl.sync_status() == "BL_OK"
