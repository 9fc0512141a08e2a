"""The next steps after the indexer proper, on the GPU through the C ABI:
Reuse with backfill and the window union, bit for bit against the oracle on
integer inputs (every score exact, so every choice is the oracle's)."""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import assert_rows_exact, seq_of, to_device

pytestmark = pytest.mark.gpu

F32 = gen.F32


@pytest.fixture(scope="module")
def tiny():
    cfg = gen.WORKLOADS["tiny_int_prefill"]
    p = gen.make_prefill(cfg["L"], cfg["H"], cfg["D"], F32, kind="int", seed=0)
    return p, to_device(p), cfg


@pytest.mark.parametrize("g,C,kk", [(4, 256, 64), (8, 100, 37), (1, 64, 64), (2, 40, 9)])
def test_reuse_backfill_exact(tiny, g, C, kk):
    """Power-of-two member counts keep the integer proxy dyadic (exact fp32 scores), so
    candidates and proxy scores are the oracle's bit for bit."""
    p, dev, _ = tiny
    seq = seq_of(dev)
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
    bf = pv.reuse_backfill(0, p.L, g, cand, cs, kk)
    reu = pv.reuse(0, p.L, g, cand, kk)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    q, qs, w, k, ks = p.codes()
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    ocand, ocs = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, p.L, g, C, kk)
    assert_rows_exact(cand.cpu(), ocand, "cand")
    assert_rows_exact(bf.cpu(), oracle.reuse_backfill(p.L, g, ocand, ocs, kk), "backfill")
    # where nothing of the proxy's top-k lies after the member, it is Reuse
    c = ocand[:, :kk]
    t = np.arange(p.L)
    unmasked = (c[t // g] <= t[:, None]).all(axis=1)
    assert unmasked.any()
    assert (bf.cpu().numpy()[unmasked] == reu.cpu().numpy()[unmasked]).all()


def test_reuse_backfill_row_range(tiny):
    """Rows [t0, t1) with candidate rows relative to t0 / g match the full call."""
    p, dev, _ = tiny
    g, C, kk = 4, 128, 32
    seq = seq_of(dev)
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
    full = pv.reuse_backfill(0, p.L, g, cand, cs, kk)
    t0, t1 = 200, 517
    part = pv.reuse_backfill(t0, t1, g, cand[t0 // g:], cs[t0 // g:], kk)
    torch.cuda.synchronize()
    assert (part.cpu() == full.cpu()[t0:t1]).all()


@pytest.mark.parametrize("window", [1, 3, 64, 300])
def test_window_union_exact(tiny, window):
    p, dev, cfg = tiny
    kk = cfg["topk"]
    idx, _ = pv.dense_index(seq_of(dev), kk)
    out = pv.window_union(idx, window)
    torch.cuda.synchronize()
    q, qs, w, k, ks = p.codes()
    oidx, _ = oracle.dense_index(F32, q, qs, w, k, ks, kk)
    assert (out.cpu().numpy() == oracle.window_union_rows(oidx, 0, window)).all()


def test_window_union_explicit_positions():
    """Decode-style rows: positions given per row (one negative: no row)."""
    rng = np.random.default_rng(4)
    rows, kk, window = 7, 16, 5
    pos = np.array([0, 3, 40, 41, 1000, -1, 17], dtype=np.int32)
    idx = np.full((rows, kk), -1, dtype=np.int32)
    for r, t in enumerate(pos):
        if t < 0:
            continue
        n = min(kk, t + 1)
        idx[r, :n] = np.sort(rng.choice(t + 1, n, replace=False))
    out = pv.window_union(torch.from_numpy(idx).cuda(), window,
                          positions=torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for r, t in enumerate(pos):
        if t < 0:
            assert (got[r] == -1).all()
            continue
        sel = idx[r][idx[r] >= 0]
        u = oracle.window_union(sel, int(t), window)
        assert got[r, :len(u)].tolist() == list(u) and (got[r, len(u):] == -1).all()


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_ragged_batch_matches_each_sequence(mode):
    """A packed batch of ragged sequences: every sequence's rows as the oracle
    computes that sequence alone (power-of-two member counts, so exact)."""
    lens = [1, 37, 300, 130, 514, 64]
    g, C, kk = 4, 64, 16
    parts = [gen.make_prefill(n, 4, 32, F32, kind="int", seed=100 + i) for i, n in enumerate(lens)]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    cat = lambda name: torch.cat([getattr(p, name) for p in parts]).cuda().contiguous()
    batch = pv.make_varlen(cu.tolist(), cat("q"), None, cat("w"), cat("k"), None)
    idx = pv.index_varlen(batch, mode, g, C, kk).cpu().numpy()
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    for i, p in enumerate(parts):
        q, qs, w, k, ks = p.codes()
        got = idx[cu[i]:cu[i + 1]]
        if mode == 0:
            want, _ = oracle.dense_index(F32, q, qs, w, k, ks, kk)
        else:
            opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
            ocand, _ = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, p.L, g, C, kk)
            want = (oracle.reuse(p.L, g, ocand, kk) if mode == 1 else
                    oracle.refine(F32, q, qs, w, k, ks, g, ocand, kk)[0])
        assert_rows_exact(got, want, f"sequence {i} (L={p.L}) mode {mode}")


def _ragged(lens, dtype, seed):
    """A packed batch of sequences of the given lengths (0 allowed), DSA-like
    inputs at H = 64, D = 128, and each sequence's own device tensors."""
    parts = {i: gen.make_prefill(n, 64, 128, dtype, kind="dsa", seed=seed + i)
             for i, n in enumerate(lens) if n > 0}
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)

    def cat(name):
        xs = [getattr(parts[i], name) for i in sorted(parts)]
        return None if xs[0] is None else torch.cat(xs).cuda().contiguous()

    batch = pv.make_varlen(cu.tolist(), cat("q"), cat("q_scale"), cat("w"), cat("k"),
                           cat("k_scale"))
    return batch, cu, {i: to_device(p) for i, p in parts.items()}


def _alone(dev, mode, g, C, kk):
    seq = seq_of(dev)
    if mode == 0:
        return pv.dense_index(seq, kk)[0]
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)[0]
    if mode == 1:
        return pv.reuse(0, dev["q"].shape[0], g, cand, kk)
    return pv.refine(seq, g, cand, kk)[0]


@pytest.mark.parametrize("dtype,mode,cap", [(gen.E4M3, 0, 0), (gen.E4M3, 1, 0), (gen.E4M3, 2, 0),
                                            (gen.E4M3, 0, 1 << 20), (gen.E4M3, 1, 1 << 20),
                                            (gen.E4M3, 2, 1 << 20), (gen.BF16, 2, 0),
                                            (gen.BF16, 0, 600 << 10)])
def test_ragged_one_launch_equals_each_sequence_alone(dtype, mode, cap):
    """The one-launch ragged batch (tensor-core shapes) against each sequence
    run alone through the single-sequence calls: bit for bit, with empty and
    one-token sequences, groups cut by sequence ends, and (cap set) score
    buffers so small that launches cut row blocks."""
    lens = [0, 1, 7, 8, 9, 300, 0, 1000, 2049, 130, 64, 3]
    g, C, kk = 8, 512, 128
    batch, cu, devs = _ragged(lens, dtype, seed=500)
    if cap:
        assert pv.pivot_set_score_buffer_cap(cap) == 0
    try:
        idx = pv.index_varlen(batch, mode, g, C, kk)
        torch.cuda.synchronize()
        assert pv.device_error() == 0
        got = idx.cpu().numpy()
        for i, dev in devs.items():
            want = _alone(dev, mode, g, C, kk).cpu().numpy()
            assert_rows_exact(got[cu[i]:cu[i + 1]], want, f"sequence {i} (L={lens[i]}) mode {mode}")
    finally:
        pv.pivot_set_score_buffer_cap(0)


def test_ragged_one_launch_launch_count():
    """Many short sequences take a fixed number of launches, not a few per
    sequence."""
    lens = [64] * 48
    batch, _, _ = _ragged(lens, gen.E4M3, seed=900)
    ws = torch.empty(pv.pivot_index_varlen_workspace_size(batch, 2, 8, 256, 64),
                     dtype=torch.uint8, device="cuda")
    pv.index_varlen(batch, 2, 8, 256, 64, ws=ws)
    torch.cuda.synchronize()
    n0 = pv.pivot_launch_count()
    pv.index_varlen(batch, 2, 8, 256, 64, ws=ws)
    torch.cuda.synchronize()
    assert pv.pivot_launch_count() - n0 <= 12


@pytest.mark.parametrize("mode,window", [(0, 1), (0, 5), (0, 64), (1, 5), (2, 5), (2, 64)])
def test_window_outside_exact(tiny, mode, window):
    """The window kept out of the candidates, then added: bit for bit."""
    p, dev, cfg = tiny
    g, C, kk = cfg["g"], cfg["C"], cfg["topk"]
    out = pv.index_window_outside(seq_of(dev), mode, g, C, kk, window)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    q, qs, w, k, ks = p.codes()
    want = oracle.index_window_outside(F32, q, qs, w, k, ks, mode, g, C, kk, window)
    assert_rows_exact(out.cpu(), want, f"window outside mode {mode} w={window}")
