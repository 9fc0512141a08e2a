"""Rank-ordered index rows (PIVOT_ORDER_RANK) through the C ABI.

A rank-ordered row lists the selected positions by score, highest first,
and equal scores by position, lowest first (the tie rule of the selection
itself, "Sparse Attention의 Indexer", Fig. 1-2: top-k keeps the highest
scores).  On integer-valued inputs every score is exact, so the GPU rows
must equal the oracle's selection sorted by (score descending, position
ascending), element by element.  On real-valued inputs the row must hold
exactly the set the position-ordered call returns, its scores must not
increase along the row, and equal scores must come by position.
"""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import assert_rows_exact, to_device

pytestmark = pytest.mark.gpu

F32, BF16, E4M3 = gen.F32, gen.BF16, gen.E4M3
RANK = pv.ORDER_RANK


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


def _seq(dev, order, t_begin=0, t_end=0):
    return pv.make_seq(dev["q"], dev["q_scale"], dev["w"], dev["k"], dev["k_scale"], t_begin,
                       t_end, order=order)


def rank_sorted(idx, sc):
    """Oracle rows (positions, fp64 scores) re-listed in rank order."""
    idx = np.asarray(idx)
    sc = np.asarray(sc)
    out_i = np.full_like(idx, -1)
    out_s = np.full(sc.shape, -np.inf)
    for r in range(idx.shape[0]):
        ok = idx[r] >= 0
        pos, s = idx[r][ok], sc[r][ok]
        o = np.lexsort((pos, -s))
        out_i[r, :len(o)] = pos[o]
        out_s[r, :len(o)] = s[o]
    return out_i, out_s


def _rank_consistent(idx, sc, pos_idx, what):
    """Real-valued rows: same set as the position-ordered call, scores non-
    increasing along the row, equal scores listed by position."""
    idx, sc, pos_idx = (np.asarray(x) for x in (idx, sc, pos_idx))
    for r in range(idx.shape[0]):
        ok = idx[r] >= 0
        assert (np.sort(idx[r][ok]) == pos_idx[r][pos_idx[r] >= 0]).all(), (what, r)
        s = sc[r][ok]
        assert (np.diff(s) <= 0).all(), (what, r)
        same = np.diff(s) == 0
        assert (np.diff(idx[r][ok])[same] > 0).all(), (what, r)
        assert (idx[r][~ok] == -1).all() and ok[:ok.sum()].all(), (what, r)


def test_tiny_integer_rank_order_exact():
    cfg = gen.WORKLOADS["tiny_int_prefill"]
    p = gen.make_prefill(cfg["L"], cfg["H"], cfg["D"], F32, kind="int", seed=0)
    dev = to_device(p)
    g, C, kk = cfg["g"], cfg["C"], cfg["topk"]
    q, qs, w, k, ks = p.codes()
    seq = _seq(dev, RANK)
    idx, sc = pv.dense_index(seq, kk, with_score=True)
    oi, os_ = rank_sorted(*oracle.dense_index(F32, q, qs, w, k, ks, kk))
    assert_rows_exact(idx.cpu(), oi, "dense rank")
    ok = oi >= 0
    assert (sc.cpu().numpy()[ok] == os_[ok]).all()

    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    ocand, ocs = rank_sorted(*oracle.proxy_scan(F32, opq, opqs, opw, k, ks, p.L, g, C, kk))
    assert_rows_exact(cand.cpu(), ocand, "cand rank")
    assert (cs.cpu().numpy()[ocand >= 0] == ocs[ocand >= 0]).all()
    # Reuse keeps the candidates' order: the proxy's top-k by rank, masked
    reu = pv.reuse(0, p.L, g, cand, kk)
    assert_rows_exact(reu.cpu(), oracle.reuse(p.L, g, ocand, kk), "reuse rank")
    ref, rs = pv.refine(seq, g, cand, kk, with_score=True)
    oref, ors = rank_sorted(*oracle.refine(F32, q, qs, w, k, ks, g, ocand, kk))
    assert_rows_exact(ref.cpu(), oref, "refine rank")
    torch.cuda.synchronize()
    assert pv.device_error() == 0


@pytest.mark.parametrize("L,kk", [(6000, 100), (3000, 2048)])
def test_long_integer_rows_rank_order_exact(L, kk):
    """Rows past the fast path's buffer (sampled bound) and k = 2048 (the
    configurations' k) with heavy ties: still the oracle's order exactly."""
    p = gen.make_prefill(L, 4, 32, F32, kind="int", seed=L + 3)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 40).astype(int)) | {kk - 1, kk, L - 1}))
    idx, sc = pv.dense_index(_seq(dev, RANK), kk, with_score=True)
    oi, os_ = rank_sorted(*oracle.dense_index(F32, q, qs, w, k, ks, kk, rows=rows))
    assert_rows_exact(idx.cpu().numpy()[rows], oi, "dense rank long")
    got = sc.cpu().numpy()[rows]
    assert (got[oi >= 0] == os_[oi >= 0]).all()


@pytest.mark.parametrize("dtype", [BF16, E4M3])
def test_real_valued_rank_rows_hold_the_position_rows(dtype):
    L, H, D, g, C, kk = 1500, 64, 128, 8, 384, 128
    p = gen.make_prefill(L, H, D, dtype, kind="dsa", seed=7)
    dev = to_device(p)
    a_idx, _ = pv.dense_index(_seq(dev, pv.ORDER_POSITION), kk)
    r_idx, r_sc = pv.dense_index(_seq(dev, RANK), kk, with_score=True)
    _rank_consistent(r_idx.cpu(), r_sc.cpu(), a_idx.cpu(), "dense")
    for order in (pv.ORDER_POSITION, RANK):
        seq = _seq(dev, order)
        pq, pqs, pw = pv.proxy_reduce(seq, g)
        cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
        ref, rs = pv.refine(seq, g, cand, kk, with_score=True)
        if order == pv.ORDER_POSITION:
            a_cand, a_ref = cand.cpu().numpy(), ref.cpu().numpy()
            continue
        _rank_consistent(cand.cpu(), cs.cpu(), np.sort(a_cand, axis=1), "cand")
        # the first k of a rank-ordered candidate row are the proxy's top-k
        assert (np.sort(cand.cpu().numpy()[:, :kk], axis=1) == np.sort(a_cand[:, :kk], axis=1)).all()
        _rank_consistent(ref.cpu(), rs.cpu(), a_ref, "refine")
    torch.cuda.synchronize()
    assert pv.device_error() == 0


def test_decode_integer_rank_order_exact():
    Gm = 2
    d = gen.make_decode(B=3, Gm=Gm, H=4, D=32, dtype=F32, len_lo=50, len_hi=700, seed=9)
    gg = torch.Generator().manual_seed(5)
    d.q = torch.randint(-3, 4, d.q.shape, generator=gg).float()
    d.kc = torch.randint(-3, 4, d.kc.shape, generator=gg).float()
    d.w = torch.randint(1, 5, d.w.shape, generator=gg).float()
    c = "cuda"
    batch = pv.make_decode(d.q.to(c), None, d.w.to(c), d.kc.to(c), None, d.cache_len.to(c),
                           order=RANK)
    q, qs, w, kc, kcs, cl = d.codes()
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        idx, cand = pv.decode(batch, mode, 128, 32, want_cand=True)
        oidx, ocand, osc = oracle.decode(F32, q, qs, w, kc, kcs, cl, mode, 128, 32)
        if mode == pv.DENSE:
            oi, _ = rank_sorted(oidx.reshape(-1, 32), osc.reshape(-1, 32))
            assert_rows_exact(idx.cpu().reshape(-1, 32), oi, "decode dense rank")
        else:
            # candidates: the oracle's set by proxy score, rank-ordered
            gc = cand.cpu().numpy()
            for b in range(3):
                pq, pqs, pw = oracle.proxy_reduce(F32, q[b], None, w[b], Gm)
                ok = ocand[b] >= 0
                s = oracle.score_positions(F32, pq, pqs, pw, kc[b], None, 0, ocand[b][ok])
                oc, _ = rank_sorted(ocand[b][None, ok], s[None, :])
                assert (gc[b][:ok.sum()] == oc[0]).all(), ("decode cand rank", b)
            if mode == pv.REUSE:
                for b in range(3):
                    for m in range(Gm):
                        lim = int(cl[b]) - Gm + m
                        want = [x for x in gc[b][:32] if 0 <= x <= lim]
                        want += [-1] * (32 - len(want))
                        assert list(idx.cpu().numpy()[b][m]) == want
    torch.cuda.synchronize()
    assert pv.device_error() == 0


def test_ragged_batch_rank_order_matches_each_sequence():
    """The one-launch ragged batch in rank order equals each sequence run
    alone in rank order (FP8, H = 64, D = 128), three modes."""
    lens = [0, 1, 9, 700, 2100, 130]
    H, D, g, C, kk = 64, 128, 8, 512, 128
    parts = [gen.make_prefill(max(n, 1), H, D, E4M3, kind="dsa", seed=50 + i)
             for i, n in enumerate(lens)]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    cat = lambda xs: torch.cat(xs).cuda()  # noqa: E731
    q = cat([pp.q[:n] for pp, n in zip(parts, lens)])
    qs = cat([pp.q_scale[:n] for pp, n in zip(parts, lens)])
    w = cat([pp.w[:n] for pp, n in zip(parts, lens)])
    k = cat([pp.k[:n] for pp, n in zip(parts, lens)])
    ks = cat([pp.k_scale[:n] for pp, n in zip(parts, lens)])
    batch = pv.make_varlen(cu, q, qs, w, k, ks, order=RANK)
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        got = pv.index_varlen(batch, mode, g, C, kk)
        for i, n in enumerate(lens):
            if n == 0:
                continue
            a, b = cu[i], cu[i + 1]
            seq = pv.make_seq(q[a:b], qs[a:b], w[a:b], k[a:b], ks[a:b], order=RANK)
            if mode == pv.DENSE:
                want, _ = pv.dense_index(seq, kk)
            else:
                pq, pqs, pw = pv.proxy_reduce(seq, g)
                cand, _ = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)
                want = (pv.reuse(0, n, g, cand, kk) if mode == pv.REUSE
                        else pv.refine(seq, g, cand, kk)[0])
            assert torch.equal(got[a:b], want), (mode, i)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
