"""The N > 1 host logic on CPU: world-size-2 gloo process groups.

Covers the row sharding of one sequence across ranks (ranges cover every
query once, causal work balanced) and the benchmark's rank plumbing (each
rank's rows are its zig-zag ranges of the one sequence, timings reduce to
the max over ranks, whole-job value)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from top_token_selection_b200.sharding import (causal_work, varlen_shards, varlen_subbatch,
                                                zigzag_ranges)


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
        rows = [None] * world
        dist.all_gather_object(rows, bench.rank_rows(L, g, world, rank))
        q.put((rank, gathered, t_max, rows, bench.dist_env()))
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
    assert res[0][3] == gathered                               # the bench's rows are these
    assert res[0][4] == (0, 0, 2) and res[1][4] == (1, 1, 2)


def test_job_value_is_whole_job():
    import bench
    # one sequence of 131072 queries x 5 steps in 1000 ms (slowest rank)
    assert bench.job_value(131072, 1000.0, 5) == pytest.approx(131072 * 5)
    assert bench.rank_rows(1000, 8, 1, 0) == [(0, 1000)]


def test_single_rank_ranges_are_the_whole_sequence():
    assert zigzag_ranges(100, 8, 1, 0) == [(0, 100)]
    with pytest.raises(ValueError):
        zigzag_ranges(100, 8, 2, 2)


def _varlen_worker(rank, world, port, cu, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = varlen_shards(cu, world)[rank]
        sub_cu, spans = varlen_subbatch(cu, mine)
        # each rank "indexes" its sub-batch: row t of a sequence gets the
        # value (sequence start + t), written back through its span
        rows = torch.full((cu[-1],), -1, dtype=torch.int64)
        for (a, b), s0 in zip(spans, sub_cu[:-1]):
            rows[a:b] = torch.arange(a, b)
        dist.all_reduce(rows, op=dist.ReduceOp.MAX)   # only to check the pieces on CPU
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        q.put((rank, gathered, rows.tolist(), sub_cu))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [[3000, 5, 0, 1, 700, 700, 64, 2048, 9, 0, 130, 1500],
                                  [256] * 37, [1, 0, 0, 2]])
def test_two_rank_ragged_batch_shards_by_sequence(lens):
    """Whole sequences per rank: every token's row comes from exactly one
    rank, both ranks agree on the split, causal work is balanced."""
    world = 2
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_varlen_worker, args=(r, world, port, cu, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert res[0][1] == res[1][1]
    shards = res[0][1]
    seqs = sorted(i for s in shards for i in s)
    assert seqs == [i for i, n in enumerate(lens) if n > 0]          # each sequence once
    assert res[0][2] == list(range(cu[-1]))                          # every row written back
    for rank in range(world):
        assert res[rank][3][-1] == sum(lens[i] for i in shards[rank])
    work = [sum(lens[i] * (lens[i] + 1) // 2 for i in s) for s in shards]
    longest = max(n * (n + 1) // 2 for n in lens)
    assert max(work) - min(work) <= longest                         # greedy bound
    if len(set(lens)) == 1:
        assert abs(len(shards[0]) - len(shards[1])) <= 1


def test_varlen_shards_single_rank_and_errors():
    assert varlen_shards([0, 3, 3, 10], 1) == [[0, 2]]
    assert varlen_shards([0], 2) == [[], []]
    with pytest.raises(ValueError):
        varlen_shards([0, 5, 3], 2)
