"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by independent work: each rank runs its own seeded
replica of the workload, or (--shard heads) its own range of one workload's
heads; there is no data-path collective.  What crosses ranks is only the
timing reduction: the barrier, the max of the per-rank times and the sum of
the per-rank work.  These run here as two gloo processes, with the head
partition.
"""
from __future__ import annotations

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.init_dist(world, "gloo")
    bench.barrier(world)
    mx = bench.max_over_ranks(10.0 + rank, world)
    sm = bench.sum_over_ranks(1.5 * (rank + 1), world)
    # each rank's replica gets its own seed: inputs differ across ranks
    from temporal_block_sparse_sm_b200 import synthetic
    cfg = synthetic.WorkloadConfig("t", 1, 1, 64, 64, 64, 64, (1, 8, 8), 1, 0.05, 0.0)
    q0 = synthetic.Workload(cfg, seed=rank).inputs(0)[0].float()
    import torch
    import torch.distributed as dist
    gathered = [torch.zeros_like(q0) for _ in range(world)]
    dist.all_gather(gathered, q0)
    distinct = not torch.equal(gathered[0], gathered[1])
    # head sharding: the ranks' head ranges tile [0, H) exactly, for several H
    covers = []
    for H in (1, 2, 3, 12, 24):
        if world > H:
            continue
        h0, h1 = bench.head_range(rank, world, H)
        rng = torch.tensor([h0, h1], dtype=torch.int64)
        got = [torch.zeros_like(rng) for _ in range(world)]
        dist.all_gather(got, rng)
        heads = [h for r in got for h in range(int(r[0]), int(r[1]))]
        covers.append(heads == list(range(H)) and all(int(r[1]) > int(r[0]) for r in got))
    dist.destroy_process_group()
    q.put((rank, mx, sm, distinct, all(covers)))


def test_timing_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, distinct, covers in res:
        assert mx == 11.0
        assert sm == 1.5 + 3.0
        assert distinct
        assert covers


@pytest.mark.parametrize("H", [1, 5, 12, 24])
def test_head_ranges_tile_the_heads(H):
    import bench
    for world in range(1, H + 1):
        ranges = [bench.head_range(r, world, H) for r in range(world)]
        assert [h for a, b in ranges for h in range(a, b)] == list(range(H))
        sizes = [b - a for a, b in ranges]
        assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1


def test_single_rank_reductions_are_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.sum_over_ranks(3.0, 1) == 3.0
    bench.barrier(1)
