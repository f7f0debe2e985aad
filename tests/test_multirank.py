"""Host logic of the multi-GPU paths, run as world-size-2 gloo ranks on the
CPU.  Replicas (the benchmark's default): every rank runs its own copy of the
workload (no data-path collective); the step time is the maximum over ranks
and the throughput counts every rank's work.  Head sharding
(softmax_cast_precision_b200.parallel): the kv heads are partitioned across
ranks and one all-gather assembles every head's output on every rank."""
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


def test_kv_head_ranges_partition_the_heads():
    import sys

    sys.path.insert(0, ROOT)
    from softmax_cast_precision_b200.parallel import kv_head_range

    for Hkv in (1, 2, 3, 8, 13):
        for world in (1, 2, 3, 4, 8):
            ranges = [kv_head_range(Hkv, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [r1 - r0 for r0, r1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        kv_head_range(4, 2, 2)


def _fake_compute(q, k, v, *, causal, p_scale, kv_order):
    """A stand-in for one shard's forward pass: o and lse encode the query head
    each output row came from (q[..., 0] holds the global head index)."""
    import torch

    o = q[..., :1].float().expand(-1, -1, -1, q.shape[-1]).to(torch.bfloat16) + 0 * k.sum()
    lse = q[..., 0].float() * 2.0
    return o, lse


def _sharded_rank_main(rank, world, port, out, H, Hkv):
    import datetime
    import sys

    import torch
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    from softmax_cast_precision_b200.parallel import fwd_head_sharded

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        B, N, d = 2, 3, 4
        q = torch.arange(H, dtype=torch.float32).view(1, H, 1, 1).expand(B, H, N, d).contiguous()
        k = torch.zeros((B, Hkv, N, d))
        v = torch.zeros((B, Hkv, N, d))
        o, lse = fwd_head_sharded(q, k, v, causal=True, group=None, compute=_fake_compute)
        out[rank] = (o.float().tolist(), lse.tolist())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H,Hkv", [(4, 4), (6, 3), (8, 2), (3, 1)])
def test_head_sharded_forward_assembles_every_head(H, Hkv):
    import torch

    ctx = mp.get_context("spawn")
    world = 2
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_sharded_rank_main, args=(r, world, port, out, H, Hkv)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        o = torch.tensor(res[r][0])
        lse = torch.tensor(res[r][1])
        assert o.shape == (2, H, 3, 4) and lse.shape == (2, H, 3)
        for h in range(H):
            assert torch.all(o[:, h] == h) and torch.all(lse[:, h] == 2 * h)
