"""Host side of the multi-GPU benchmark path, run as two gloo ranks on the CPU:
the job time is the slowest rank's and the whole-job rate counts every rank's
work (weak scaling, no collective on the data path)."""
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


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 100.0 + 25.0 * rank             # ranks finish at different times
        worst = bench.max_over_ranks(my_ms, world)
        bench.barrier(world)
        rate = bench.job_throughput(world, 16384, 10, worst)
        out[rank] = (worst, rate)
    finally:
        dist.destroy_process_group()


def test_two_ranks_slowest_rank_and_job_rate():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        worst, rate = out[r]
        assert worst == pytest.approx(125.0)
        assert rate == pytest.approx(2 * 16384 * 10 / 0.125)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1, 100, 4, 2000.0) == pytest.approx(200.0)
