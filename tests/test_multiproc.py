"""Multi-rank host logic of bench.py with world size 2 over gloo on CPU: the max-over-
ranks timing reduction, the whole-job rate, and the sharding of independent layers for
the quantize-on-load leg.  The forward itself is replicated per GPU (no data-path
collective), so these are the only cross-rank steps."""
from __future__ import annotations

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


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        times = [10.0 + rank, 5.0 - rank, 7.5]
        mx = bench.max_over_ranks(times)
        sm = bench.sum_over_ranks([1.0 + rank])
        layers = list(bench.shard_range(48, rank, world))
        all_layers = [None] * world
        dist.all_gather_object(all_layers, layers)
        rate = bench.aggregate_rate([100.0] * world, mx[0])
        q.put((rank, mx, sm, all_layers, rate))
    finally:
        dist.destroy_process_group()


def test_two_rank_reductions_and_sharding():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, all_layers, rate in res:
        assert mx == [11.0, 5.0, 7.5]           # element-wise max over the two ranks
        assert sm == [3.0]
        flat = [l for part in all_layers for l in part]
        assert sorted(flat) == list(range(48)) and len(flat) == 48   # disjoint, complete
        assert abs(rate - 200.0 / 11.0) < 1e-12  # all ranks' units over the slowest time


@pytest.mark.parametrize("n,world", [(48, 1), (48, 5), (7, 8), (0, 3)])
def test_shard_range_partition(n, world):
    import bench
    parts = [list(bench.shard_range(n, r, world)) for r in range(world)]
    flat = [x for p in parts for x in p]
    assert flat == list(range(n))
    sizes = [len(p) for p in parts]
    assert max(sizes) - min(sizes) <= 1
