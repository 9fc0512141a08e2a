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


def varlen_shards(cu_seqlens, world: int):
    """Whole sequences of a ragged batch per rank, balancing causal work.

    Sequences are independent (each has its own keys), so a packed batch
    shards by sequence with no exchange step.  Sequence i costs
    len_i (len_i + 1) / 2 causal pairs; sequences are dealt longest first to
    the rank with the least work so far (ties to the lower rank), which
    keeps every rank within the longest sequence's cost of the mean.  A
    sequence much longer than the rest is better split by rows with
    ``zigzag_ranges`` and the single-sequence calls.  Returns one ascending
    list of sequence indices per rank (empty sequences go nowhere)."""
    n = len(cu_seqlens) - 1
    if world < 1 or n < 0:
        raise ValueError("bad arguments")
    lens = [int(cu_seqlens[i + 1]) - int(cu_seqlens[i]) for i in range(n)]
    if any(x < 0 for x in lens):
        raise ValueError("cu_seqlens must not decrease")
    order = sorted((i for i in range(n) if lens[i] > 0), key=lambda i: (-lens[i], i))
    load = [0] * world
    out = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda x: (load[x], x))
        out[r].append(i)
        load[r] += lens[i] * (lens[i] + 1) // 2
    return [sorted(s) for s in out]


def varlen_subbatch(cu_seqlens, seqs):
    """A rank's sub-batch: its cu_seqlens and, per sequence, the token range
    [a, b) of the full packed batch its rows come from (and go back to)."""
    cu = [0]
    spans = []
    for i in seqs:
        a, b = int(cu_seqlens[i]), int(cu_seqlens[i + 1])
        spans.append((a, b))
        cu.append(cu[-1] + b - a)
    return cu, spans
