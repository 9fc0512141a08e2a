"""Splitting one prefill sequence's queries across ranks.

Groups are independent once the keys are known (abstract of arXiv
2607.24593: one full-prefix scan per group), so a sequence's query rows can
be indexed by several GPUs, each holding the whole key array and calling
the library on its own row ranges (``pivot_seq_t.t_begin/t_end``).  There
is no exchange step: each rank writes the index rows of its own ranges.

Causal work grows with position, so contiguous equal splits are unbalanced.
``zigzag_ranges`` cuts the groups into 2*world equal blocks and gives rank r
blocks r and 2*world-1-r: an early (cheap) and a late (costly) block.
"""
from __future__ import annotations


def zigzag_ranges(L: int, g: int, world: int, rank: int):
    """Row ranges [(t_begin, t_end), ...] of `rank`, group-aligned."""
    if not (0 <= rank < world) or L < 1 or g < 1:
        raise ValueError("bad arguments")
    G = -(-L // g)
    nb = 2 * world
    bounds = [(i * G) // nb for i in range(nb + 1)]
    out = []
    for blk in sorted({rank, nb - 1 - rank}):
        j0, j1 = bounds[blk], bounds[blk + 1]
        if j0 < j1:
            lo, hi = j0 * g, min(L, j1 * g)
            if out and out[-1][1] == lo:     # adjacent blocks: one range
                out[-1] = (out[-1][0], hi)
            else:
                out.append((lo, hi))
    return out


def causal_work(ranges):
    """Sum over rows t of (t + 1): the dense indexer's pairs for those rows."""
    return sum((b * (b + 1) - a * (a + 1)) // 2 for a, b in ranges)
