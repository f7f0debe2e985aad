"""Host logic of the multi-GPU benchmark path, run as world-size-2 gloo ranks
on the CPU: every rank runs its own copy of the workload (no data-path
collective); the step time is the maximum over ranks and the throughput
counts every rank's work."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime
    import sys

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        value = bench.aggregate_throughput(1e12, world, worst)
        out[rank] = (worst, value, bench.rank_seed(rank))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_aggregation():
    ctx = mp.get_context("spawn")
    world = 2
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        worst, value, seed = res[r]
        assert worst == 15.0  # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 1e12 / 15e-3 / 1e12)
    assert res[0][2] != res[1][2]  # independent inputs per rank


def test_single_rank_is_identity():
    import sys

    import torch

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.aggregate_throughput(8.0e12, 1, 8.0) == pytest.approx(1000.0)
