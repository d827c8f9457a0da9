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


def test_stage_rooflines_of_the_main_workload():
    """Per-stage rooflines from stage times: bytes or flops of the flop model
    over the time, as a fraction of the given peak."""
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    from gqe_inputs import CONFIGS
    d = CONFIGS["main_b8_t2048"]
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 1000.0}
    r = bench.stage_rooflines(d, {"route": 1.0, "qproj": 1.0, "attention": 1.0, "combine": 1.0}, peaks)
    N = 8 * 2048
    # routing: x (N*D bf16) dominates: 33.5 MB in 1 ms is 33.5 GB/s
    assert r["route"]["bound"] == "hbm" and 33.5 < r["route"]["achieved"] < 37.0
    # attention of 9 row sets, causal over 2048 positions per sequence: 4*64*9*8*2048*2049/2 flop
    assert r["attention"]["algorithmic"] == 4 * 64 * 9 * 8 * 2048 * 2049 // 2
    assert abs(r["attention"]["achieved"] - r["attention"]["algorithmic"] / 1e-3 / 1e12) < 1e-9
    assert r["combine"]["algorithmic"] == 2 * N * 17 * 64 * 1024
    for v in r.values():
        assert abs(v["frac"] - v["achieved"] / 1000.0) < 1e-12
