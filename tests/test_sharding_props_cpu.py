"""Properties of the host-side sharding, over random inputs (hypothesis):
every query row / sequence is assigned exactly once, group alignment holds,
and the causal work stays balanced within the stated bounds."""
from hypothesis import given, settings, strategies as st

from top_token_selection_b200.sharding import (causal_work, varlen_shards, varlen_subbatch,
                                               zigzag_ranges)


@settings(max_examples=200, deadline=None)
@given(L=st.integers(1, 50000), g=st.integers(1, 16), world=st.integers(1, 8))
def test_zigzag_covers_each_row_once_group_aligned(L, g, world):
    seen = []
    for r in range(world):
        for a, b in zigzag_ranges(L, g, world, r):
            assert 0 <= a < b <= L
            assert a % g == 0 and (b % g == 0 or b == L)
            seen.append((a, b))
    seen.sort()
    assert seen[0][0] == 0 and seen[-1][1] == L
    for (a0, b0), (a1, b1) in zip(seen, seen[1:]):
        assert b0 == a1                                  # no gap, no overlap


@settings(max_examples=100, deadline=None)
@given(L=st.integers(20000, 200000), world=st.integers(2, 8))
def test_zigzag_balances_causal_work(L, world):
    w = [causal_work(zigzag_ranges(L, 8, world, r)) for r in range(world)]
    assert max(w) / min(w) < 1.05


@settings(max_examples=200, deadline=None)
@given(lens=st.lists(st.integers(0, 5000), min_size=0, max_size=60), world=st.integers(1, 8))
def test_varlen_shards_each_sequence_once_and_balanced(lens, world):
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    shards = varlen_shards(cu, world)
    assert len(shards) == world
    got = sorted(i for s in shards for i in s)
    assert got == [i for i, n in enumerate(lens) if n > 0]
    work = [sum(lens[i] * (lens[i] + 1) // 2 for i in s) for s in shards]
    if any(lens):
        longest = max(n * (n + 1) // 2 for n in lens)
        assert max(work) - min(work) <= longest          # the greedy bound
    for s in shards:
        sub_cu, spans = varlen_subbatch(cu, s)
        assert sub_cu[-1] == sum(b - a for a, b in spans)
        assert [b - a for a, b in spans] == [lens[i] for i in s]
