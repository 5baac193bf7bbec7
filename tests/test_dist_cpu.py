"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by independent work (each rank runs its own seeded
replica of the workload; no data-path collective).  What crosses ranks is
only the timing reduction: the barrier, the max of the per-rank times and the
sum of the per-rank work.  These run here as two gloo processes.
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
    dist.destroy_process_group()
    q.put((rank, mx, sm, distinct))


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
    for rank, mx, sm, distinct in res:
        assert mx == 11.0
        assert sm == 1.5 + 3.0
        assert distinct


def test_single_rank_reductions_are_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.sum_over_ranks(3.0, 1) == 3.0
    bench.barrier(1)
