"""The data-parallel host logic of bench.py on CPU ranks (gloo, world size 2).

Each rank draws its own batch (weak scaling: no data-path collective); the
only cross-rank step is the max-over-ranks reduction of the timed region, and
the whole-job value counts every rank's MACs over the slowest rank's time.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        p = next(workloads.problems(1, rank=rank))
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        slow = bench.max_over_ranks(ms, dist)
        value = bench.whole_job_gmacs(p.M * p.N * p.K, 100, world, slow)
        out[rank] = (float(p.W[0, 0]), slow, value)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_weak_scaling():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    w0, slow0, v0 = out[0]
    w1, slow1, v1 = out[1]
    assert w0 != w1                           # independent batches per rank
    assert slow0 == slow1 == 15.0             # both ranks see the slowest rank's time
    macs = 8 * 128 * 256
    assert v0 == v1 == pytest.approx(macs * 100 * 2 / 15e-3 / 1e9)


def test_single_rank_helpers():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_gmacs(10 ** 9, 1, 1, 1000.0) == pytest.approx(1.0)
    # rank 0 of a data-parallel run reproduces the single-GPU inputs
    import workloads
    a = next(workloads.problems(2, rank=0))
    b = next(workloads.problems(2))
    np.testing.assert_array_equal(a.W, b.W)
