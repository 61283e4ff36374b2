"""Multi-process host logic of the bench on CPU: two gloo ranks.

The forward's work items are independent, so N GPUs run N independent batches
(weak scaling) with no collective on the data path; the only collectives are a
barrier and the max-over-ranks reduction of the device timings.  This checks that
host path with world_size 2 on the gloo backend (no GPU).
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        dist.barrier()
        times = [10.0 + rank, 3.0 - rank, 7.0]
        got = bench.max_over_ranks(times, dist, torch.device("cpu"))
        value = bench.whole_job_tflops(2.0e12, world, got[0])
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, value in res:
        assert got == [11.0, 3.0, 7.0]                   # the slowest rank sets each timing
        assert value == pytest.approx(2.0e12 * 2 / 11e-3 / 1e12)


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.whole_job_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)
