"""bench.py's multi-rank arithmetic on two gloo ranks (CPU): the job time is
the slowest rank's, and throughput counts every rank's batch."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 3.0 - rank]         # rank 1 slower on the first, faster on the second
        got = bench.reduce_max(mine, world, "cpu")
        out[rank] = (got, bench.job_throughput(world, 16384, got[0] / 5))
    finally:
        dist.destroy_process_group()


def test_reduce_max_and_throughput_on_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        for r in range(2):
            got, thr = out[r]
            assert got == [11.0, 3.0]
            assert thr == pytest.approx(2 * 16384 / (11.0 / 5 / 1e3))


def test_single_rank_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.job_throughput(1, 1000, 2.0) == pytest.approx(500000.0)
