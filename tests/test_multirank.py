"""The benchmark's multi-rank host logic on CPU with gloo (world size 2).

Every (batch, head) slice is an independent problem, so ranks share no data:
the only cross-rank steps are the barrier around the timed region and the
max-over-ranks reduction of the step time.
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, _ = bench.dist_env()
    bench.init_dist(w, "gloo")
    bench.barrier(w)
    slowest = bench.max_over_ranks(1.5 + r, w)
    q.put((r, slowest, bench.shard_seed(r)))
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_draw_distinct_shards():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[1] for g in got] == [2.5, 2.5]
    assert len({g[2] for g in got}) == world


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
