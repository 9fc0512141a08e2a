"""The N > 1 host logic on CPU: world-size-2 gloo process groups.

Covers the row sharding of one sequence across ranks (ranges cover every
query once, causal work balanced) and the benchmark's rank plumbing (seeds
differ per rank, timings reduce to the max over ranks, whole-job value)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from top_token_selection_b200.sharding import causal_work, zigzag_ranges


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, L, g, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        mine = zigzag_ranges(L, g, world, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        t_mine = 10.0 + 5.0 * rank
        t_max = bench.max_over_ranks(t_mine)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(0, rank))
        q.put((rank, gathered, t_max, seeds, bench.dist_env()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("L,g", [(131072, 8), (1000, 3), (17, 4)])
def test_two_rank_sharding_and_timing(L, g):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, g, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    gathered = res[0][1]
    assert gathered == res[1][1]
    rows = sorted(r for ranges in gathered for a, b in ranges for r in range(a, b))
    assert rows == list(range(L))                              # every query exactly once
    for ranges in gathered:
        for a, b in ranges:
            assert a % g == 0 and (b % g == 0 or b == L)        # group aligned
    if L >= 1000:
        w = [causal_work(r) for r in gathered]
        assert max(w) / min(w) < 1.05                          # balanced causal work
    assert res[0][2] == res[1][2] == 15.0                      # max over ranks
    assert res[0][3][0] != res[0][3][1]                        # independent replicas
    assert res[0][4] == (0, 0, 2) and res[1][4] == (1, 1, 2)


def test_aggregate_value_is_whole_job():
    import bench
    # 2 ranks x 131072 queries x 5 steps in 1000 ms (slowest rank)
    assert bench.aggregate_value(131072, 2, 1000.0, 5) == pytest.approx(2 * 131072 * 5)


def test_single_rank_ranges_are_the_whole_sequence():
    assert zigzag_ranges(100, 8, 1, 0) == [(0, 100)]
    with pytest.raises(ValueError):
        zigzag_ranges(100, 8, 2, 2)
