"""The multi-rank path of bench.py on CPU: two gloo ranks.

Every rank runs its own copy of the workload (no collective on the data path);
the only cross-rank steps are the timing reduction (MAX of the per-rank time,
SUM of the work) and the barriers around the timed region. This runs them with
world size 2 over gloo on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.dist_barrier(world)
        t = bench.dist_max(world, 1.5 + rank)          # per-rank "time"
        w = bench.dist_sum(world, 10.0 * (rank + 1))    # per-rank "work"
        bench.dist_barrier(world)
        q.put((rank, t, w))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_time_and_work():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[1] for r in res] == [2.5, 2.5]      # slowest rank
    assert [r[2] for r in res] == [30.0, 30.0]    # all ranks' work


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.dist_max(1, 3.0) == 3.0 and bench.dist_sum(1, 4.0) == 4.0
