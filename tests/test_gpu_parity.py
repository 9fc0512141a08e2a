"""GPU path vs. the CPU oracle, through the C ABI.

Sizes span several 128-key tiles and several row blocks with ragged tails;
the tiny integer workload (L=1024, H=4, D=32, k=64, g=4, C=256) compares
bit for bit, the DSA-shaped bf16 / FP8 ones within the boundary tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import (assert_rows_close, assert_rows_exact, fp32_abs_tol, proxy_score_fn,
                    score_fn_for, seq_of, to_device)

pytestmark = pytest.mark.gpu

F32, BF16, E4M3 = gen.F32, gen.BF16, gen.E4M3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


def _pivot_gpu(p, dev, g, C, topk, with_score=True):
    seq = seq_of(dev)
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, topk, with_score=with_score)
    reu = pv.reuse(0, p.L, g, cand, topk)
    ref, rs = pv.refine(seq, g, cand, topk, with_score=with_score)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    return pq, pqs, pw, cand, cs, reu, ref, rs


# ---------------------------------------------------------------------------
# proxy reduce: bit for bit
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,kind,L,H,D,g", [
    (F32, "int", 1030, 4, 32, 4),       # ragged last group (2 members)
    (BF16, "dsa", 333, 64, 128, 8),
    (E4M3, "dsa", 333, 64, 128, 8),
    (E4M3, "dsa", 64, 64, 128, 1),      # one-member groups are copies
    (BF16, "dsa", 100, 8, 64, 3),       # g not a power of two: IEEE divide
])
def test_proxy_reduce_bit_exact(dtype, kind, L, H, D, g):
    p = gen.make_prefill(L, H, D, dtype, kind=kind, seed=1)
    dev = to_device(p)
    pq, pqs, pw = pv.proxy_reduce(seq_of(dev), g)
    q, qs, w, _, _ = p.codes()
    opq, opqs, opw = oracle.proxy_reduce(dtype, q, qs, w, g)
    assert (gen.codes_of(pq.cpu(), dtype) == opq).all()
    assert (pw.cpu().numpy() == opw).all()
    if dtype == E4M3:
        assert (pqs.cpu().numpy() == opqs).all()


# ---------------------------------------------------------------------------
# integer workload: everything bit for bit
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
    cfg = gen.WORKLOADS["tiny_int_prefill"]
    p = gen.make_prefill(cfg["L"], cfg["H"], cfg["D"], F32, kind="int", seed=0)
    return p, to_device(p), cfg


def test_tiny_dense_exact(tiny):
    p, dev, cfg = tiny
    idx, sc = pv.dense_index(seq_of(dev), cfg["topk"], with_score=True)
    q, qs, w, k, ks = p.codes()
    oidx, osc = oracle.dense_index(F32, q, qs, w, k, ks, cfg["topk"])
    assert_rows_exact(idx.cpu(), oidx, "dense")
    ok = oidx >= 0
    assert (sc.cpu().numpy()[ok] == osc[ok]).all()
    assert np.isneginf(sc.cpu().numpy()[~ok]).all()


def test_tiny_pivot_exact(tiny):
    p, dev, cfg = tiny
    g, C, kk = cfg["g"], cfg["C"], cfg["topk"]
    pq, pqs, pw, cand, cs, reu, ref, rs = _pivot_gpu(p, dev, g, C, kk)
    q, qs, w, k, ks = p.codes()
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    ocand, ocs = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, p.L, g, C, kk)
    assert_rows_exact(cand.cpu(), ocand, "proxy scan")
    ok = ocand >= 0
    assert (cs.cpu().numpy()[ok] == ocs[ok]).all()
    assert_rows_exact(reu.cpu(), oracle.reuse(p.L, g, ocand, kk), "reuse")
    oref, ors = oracle.refine(F32, q, qs, w, k, ks, g, ocand, kk)
    assert_rows_exact(ref.cpu(), oref, "refine")
    ok = oref >= 0
    assert (rs.cpu().numpy()[ok] == ors[ok]).all()


def test_tiny_invariants_on_gpu(tiny):
    """g = 1 is the dense indexer; Refine over the whole prefix is dense."""
    p, dev, cfg = tiny
    kk = cfg["topk"]
    dense, _ = pv.dense_index(seq_of(dev), kk)
    _, _, _, cand, _, reu, ref, _ = _pivot_gpu(p, dev, 1, kk, kk, with_score=False)
    assert_rows_exact(reu.cpu(), dense.cpu(), "g=1 reuse")
    assert_rows_exact(ref.cpu(), dense.cpu(), "g=1 refine")
    _, _, _, cand, _, _, ref, _ = _pivot_gpu(p, dev, 4, p.L, kk, with_score=False)
    assert_rows_exact(ref.cpu(), dense.cpu(), "C=L refine")


@pytest.mark.parametrize("L,g,C,kk", [
    (37, 4, 16, 8),          # fewer keys than a tile; prefixes shorter than k; 1-member tail
    (300, 4, 64, 64),        # C == k
    (129, 2, 300, 7),        # C larger than every prefix
    (514, 8, 40, 1),         # k = 1; 2-member tail group
    (2048, 4, 64, 16),       # one candidate tile per Refine item, several items per CTA
    (1024, 2, 128, 32),      # the same with full tiles
])
def test_edge_shapes_exact(L, g, C, kk):
    """Every group has a power-of-two member count, so the proxy mean of
    integers is dyadic, every fp32 score is exact and every comparison is
    bit for bit."""
    p = gen.make_prefill(L, 4, 32, F32, kind="int", seed=L)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    idx, _ = pv.dense_index(seq_of(dev), kk)
    assert_rows_exact(idx.cpu(), oracle.dense_index(F32, q, qs, w, k, ks, kk)[0], "dense")
    _, _, _, cand, _, reu, ref, _ = _pivot_gpu(p, dev, g, C, kk, with_score=False)
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    ocand, _ = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, L, g, C, kk)
    assert_rows_exact(cand.cpu(), ocand, "cand")
    assert_rows_exact(reu.cpu(), oracle.reuse(L, g, ocand, kk), "reuse")
    assert_rows_exact(ref.cpu(), oracle.refine(F32, q, qs, w, k, ks, g, ocand, kk)[0], "refine")


def test_long_rows_exact():
    """Rows longer than the selection's kept-entry buffer (2048 for k <= 1024)
    take the sampled-threshold path; integer scores keep it bit-exact, ties
    included."""
    L, g, C, kk = 6000, 4, 1100, 100
    p = gen.make_prefill(L, 4, 32, F32, kind="int", seed=77)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(2048, L - 1, 48).astype(int)) | {L - 1}))
    idx, sc = pv.dense_index(seq_of(dev), kk, with_score=True)
    oidx, osc = oracle.dense_index(F32, q, qs, w, k, ks, kk, rows=rows)
    assert_rows_exact(idx.cpu().numpy()[rows], oidx, "dense long rows")
    assert (sc.cpu().numpy()[rows] == osc).all()
    _, _, _, cand, _, reu, ref, _ = _pivot_gpu(p, dev, g, C, kk, with_score=False)
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    groups = np.array(sorted(set(np.linspace(600, L // g - 1, 32).astype(int))))
    ocand, _ = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
    assert_rows_exact(cand.cpu().numpy()[groups], ocand, "cand long rows")
    gc = cand.cpu().numpy()
    assert_rows_exact(ref.cpu().numpy()[rows], oracle.refine(F32, q, qs, w, k, ks, g, gc, kk,
                                                             rows=rows)[0], "refine")


@pytest.mark.parametrize("dtype", [BF16, E4M3])
def test_dsa_long_rows_within_tolerance(dtype):
    L, H, D, g, C, kk = 9000, 64, 128, 8, 2600, 300
    p = gen.make_prefill(L, H, D, dtype, kind="dsa", seed=8)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(2100, L - 1, 24).astype(int))))
    idx, sc = pv.dense_index(seq_of(dev), kk, with_score=True)
    oidx, osc = oracle.dense_index(dtype, q, qs, w, k, ks, kk, rows=rows)
    assert_rows_close(idx.cpu().numpy()[rows], oidx, osc, score_fn_for(p), rows, "dense",
                      gpu_scores=sc.cpu().numpy()[rows])
    pq, pqs, pw, cand, cs, reu, ref, rs = _pivot_gpu(p, dev, g, C, kk)
    opq, opqs, opw = oracle.proxy_reduce(dtype, q, qs, w, g)
    groups = np.array(sorted(set(np.linspace(700, L // g - 1, 16).astype(int))))
    ocand, ocs = oracle.proxy_scan(dtype, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
    assert_rows_close(cand.cpu().numpy()[groups], ocand, ocs, proxy_score_fn(p, opq, opqs, opw),
                      groups, "cand", gpu_scores=cs.cpu().numpy()[groups])


@pytest.mark.parametrize("L,g,C,kk", [(300, 5, 64, 64), (515, 3, 40, 9)])
def test_edge_shapes_odd_groups(L, g, C, kk):
    """g not a power of two: the proxy mean of integers is not dyadic, so
    proxy scores are fp32 sums of non-integers, some of them near-zero
    results of cancelling dot products at the boundary; the candidates
    compare within the relative tolerance floored by the fp32 error bound,
    and Reuse and Refine on the GPU's own candidates stay exact (members'
    own integer queries)."""
    p = gen.make_prefill(L, 4, 32, F32, kind="int", seed=L + 1)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    pq, pqs, pw, cand, cs, reu, ref, _ = _pivot_gpu(p, dev, g, C, kk)
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    assert (pq.cpu().numpy() == opq).all() and (pw.cpu().numpy() == opw).all()
    groups = np.arange(opq.shape[0])
    ocand, ocs = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, L, g, C, kk)
    assert_rows_close(cand.cpu().numpy(), ocand, ocs, proxy_score_fn(p, opq, opqs, opw), groups,
                      "cand", gpu_scores=cs.cpu().numpy(), abs_tol=fp32_abs_tol(opq, opw, k))
    gc = cand.cpu().numpy()
    assert_rows_exact(reu.cpu(), oracle.reuse(L, g, gc, kk), "reuse")
    assert_rows_exact(ref.cpu(), oracle.refine(F32, q, qs, w, k, ks, g, gc, kk)[0], "refine")


def test_f32_real_valued_within_tolerance():
    """Real-valued fp32 inputs (the DSA-shaped generator kept in fp32): the
    fp32 scores meet the relative tolerance against the fp64 oracle for
    dense, the proxy scan and Refine."""
    L, H, D, g, C, kk = 700, 4, 32, 4, 256, 64
    p = gen.make_prefill(L, H, D, F32, kind="dsa", seed=31)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 40).astype(int)) | {L - 1}))
    idx, sc = pv.dense_index(seq_of(dev), kk, with_score=True)
    oidx, osc = oracle.dense_index(F32, q, qs, w, k, ks, kk, rows=rows)
    fn = score_fn_for(p)
    assert_rows_close(idx.cpu().numpy()[rows], oidx, osc, fn, rows, "dense",
                      gpu_scores=sc.cpu().numpy()[rows])
    pq, pqs, pw, cand, cs, reu, ref, rs = _pivot_gpu(p, dev, g, C, kk)
    opq, opqs, opw = oracle.proxy_reduce(F32, q, qs, w, g)
    assert (pq.cpu().numpy() == opq).all() and (pw.cpu().numpy() == opw).all()
    groups = np.arange(opq.shape[0])
    ocand, ocs = oracle.proxy_scan(F32, opq, opqs, opw, k, ks, L, g, C, kk)
    assert_rows_close(cand.cpu().numpy(), ocand, ocs, proxy_score_fn(p, opq, opqs, opw), groups,
                      "cand", gpu_scores=cs.cpu().numpy())
    gc = cand.cpu().numpy()
    assert_rows_exact(reu.cpu(), oracle.reuse(L, g, gc, kk), "reuse")
    oref, ors = oracle.refine(F32, q, qs, w, k, ks, g, gc, kk, rows=rows)
    assert_rows_close(ref.cpu().numpy()[rows], oref, ors, fn, rows, "refine",
                      gpu_scores=rs.cpu().numpy()[rows])


def test_row_ranges_and_small_workspace_match_one_call(tiny):
    """Splitting the rows across calls (as ranks would) or forcing many
    workspace chunks changes nothing."""
    p, dev, cfg = tiny
    g, C, kk = cfg["g"], cfg["C"], cfg["topk"]
    full, _ = pv.dense_index(seq_of(dev), kk)
    a, _ = pv.dense_index(seq_of(dev, 0, 512), kk)
    b, _ = pv.dense_index(seq_of(dev, 512, 1024), kk)
    assert torch.equal(torch.cat([a, b]), full)
    small = torch.empty(64 * 1024 * 4 + 256, dtype=torch.uint8, device="cuda")
    c, _ = pv.dense_index(seq_of(dev), kk, ws=small)
    assert torch.equal(c, full)
    _, _, _, cand, _, reu, ref, _ = _pivot_gpu(p, dev, g, C, kk, with_score=False)
    seq2 = seq_of(dev, 512, 1024)
    pq, pqs, pw = pv.proxy_reduce(seq2, g)
    cand2, _ = pv.proxy_scan(seq2, g, pq, pqs, pw, C, kk)
    assert torch.equal(cand2, cand[512 // g:])
    ref2, _ = pv.refine(seq2, g, cand2, kk)
    assert torch.equal(ref2, ref[512:])
    assert torch.equal(pv.reuse(512, 1024, g, cand2, kk), reu[512:])


@pytest.mark.parametrize("world", [2, 3])
def test_zigzag_sharded_calls_match_one_call(tiny, world):
    """Each rank's zig-zag row ranges, run as separate calls (as separate
    GPUs would), reassemble the single-call result exactly."""
    from top_token_selection_b200.sharding import zigzag_ranges
    p, dev, cfg = tiny
    g, C, kk = cfg["g"], cfg["C"], cfg["topk"]
    full_dense, _ = pv.dense_index(seq_of(dev), kk)
    _, _, _, full_cand, _, full_reu, full_ref, _ = _pivot_gpu(p, dev, g, C, kk, with_score=False)
    for rank in range(world):
        for a, b in zigzag_ranges(p.L, g, world, rank):
            seq = seq_of(dev, a, b)
            d, _ = pv.dense_index(seq, kk)
            assert torch.equal(d, full_dense[a:b])
            pq, pqs, pw = pv.proxy_reduce(seq, g)
            cand, _ = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)
            assert torch.equal(cand, full_cand[a // g:-(-b // g)])
            assert torch.equal(pv.reuse(a, b, g, cand, kk), full_reu[a:b])
            r, _ = pv.refine(seq, g, cand, kk)
            assert torch.equal(r, full_ref[a:b])


# ---------------------------------------------------------------------------
# real-valued DSA-shaped inputs: bf16 and FP8
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [BF16, E4M3])
def test_dsa_small_within_tolerance(dtype):
    L, H, D, g, C, kk = 1500, 64, 128, 8, 384, 128
    p = gen.make_prefill(L, H, D, dtype, kind="dsa", seed=7)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 40).astype(int)) | {0, 1, 127, 128, L - 1}))
    idx, sc = pv.dense_index(seq_of(dev), kk, with_score=True)
    oidx, osc = oracle.dense_index(dtype, q, qs, w, k, ks, kk, rows=rows)
    fn = score_fn_for(p)
    assert_rows_close(idx.cpu().numpy()[rows], oidx, osc, fn, rows, "dense",
                      gpu_scores=sc.cpu().numpy()[rows])

    pq, pqs, pw, cand, cs, reu, ref, rs = _pivot_gpu(p, dev, g, C, kk)
    opq, opqs, opw = oracle.proxy_reduce(dtype, q, qs, w, g)
    G = opq.shape[0]
    groups = np.array(sorted(set(np.linspace(0, G - 1, 24).astype(int))))
    ocand, ocs = oracle.proxy_scan(dtype, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
    pfn = proxy_score_fn(p, opq, opqs, opw)
    assert_rows_close(cand.cpu().numpy()[groups], ocand, ocs, pfn, groups, "cand",
                      gpu_scores=cs.cpu().numpy()[groups])
    # Reuse and Refine checked on the GPU's own candidates (isolates the step)
    gcand = cand.cpu().numpy()
    assert_rows_exact(reu.cpu(), oracle.reuse(L, g, gcand, kk), "reuse")
    oref, ors = oracle.refine(dtype, q, qs, w, k, ks, g, gcand, kk, rows=rows)
    assert_rows_close(ref.cpu().numpy()[rows], oref, ors, fn, rows, "refine",
                      gpu_scores=rs.cpu().numpy()[rows])


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

def _decode_dev(d):
    c = "cuda"
    return pv.make_decode(d.q.to(c), None if d.q_scale is None else d.q_scale.to(c), d.w.to(c),
                          d.kc.to(c), None if d.kc_scale is None else d.kc_scale.to(c),
                          d.cache_len.to(c)), d


@pytest.mark.parametrize("dtype,H,D,Gm", [(BF16, 64, 128, 2), (E4M3, 64, 128, 2),
                                          (E4M3, 64, 128, 3), (BF16, 64, 128, 4)])
def test_decode_within_tolerance(dtype, H, D, Gm):
    """MTP groups of 2 (one draft token) and deeper ones (3, 4 tokens per step)."""
    d = gen.make_decode(B=5, Gm=Gm, H=H, D=D, dtype=dtype, len_lo=300, len_hi=2200, seed=3)
    batch, d = _decode_dev(d)
    q, qs, w, kc, kcs, cl = d.codes()
    C, kk = 256, 64
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        idx, cand = pv.decode(batch, mode, C, kk, want_cand=True)
        torch.cuda.synchronize()
        assert pv.device_error() == 0
        oidx, ocand, osc = oracle.decode(dtype, q, qs, w, kc, kcs, cl, mode, C, kk)
        gi = idx.cpu().numpy()
        for b in range(d.q.shape[0]):
            n = int(cl[b])
            kb = kc[b]
            kbs = None if kcs is None else kcs[b]

            def fn(m, positions, b=b, kb=kb, kbs=kbs):
                return oracle.score_positions(dtype, q[b], None if qs is None else qs[b], w[b],
                                              kb, kbs, m, positions)
            if mode == pv.DENSE:
                assert_rows_close(gi[b], oidx[b], osc[b], fn, list(range(Gm)),
                                  f"decode dense b={b}")
            else:
                gc = cand.cpu().numpy()
                if mode == pv.REUSE:
                    for m in range(Gm):
                        lim = n - Gm + m
                        want = [x for x in gc[b][:kk] if 0 <= x <= lim]
                        want += [-1] * (kk - len(want))
                        assert list(gi[b][m]) == want
                else:
                    # refine on the GPU's candidates, member by member
                    for m in range(Gm):
                        lim = n - Gm + m
                        pos = np.array([x for x in gc[b] if 0 <= x <= lim], dtype=np.int32)
                        sc = fn(m, pos)
                        order = np.lexsort((pos, -sc))[:kk]
                        ref = list(pos[order]) + [-1] * (kk - len(order))
                        refsc = list(sc[order])
                        assert_rows_close(gi[b][m:m + 1], np.array([ref]), np.array([refsc]),
                                          fn, [m], f"decode refine b={b}")


@pytest.mark.parametrize("Gm", [2, 4])
def test_decode_integer_exact(Gm):
    d = gen.make_decode(B=3, Gm=Gm, H=4, D=32, dtype=F32, len_lo=50, len_hi=700, seed=9)
    # integer-valued keys and queries for exact comparison
    gg = torch.Generator().manual_seed(5)
    d.q = torch.randint(-3, 4, d.q.shape, generator=gg).float()
    d.kc = torch.randint(-3, 4, d.kc.shape, generator=gg).float()
    d.w = torch.randint(1, 5, d.w.shape, generator=gg).float()
    batch, d = _decode_dev(d)
    q, qs, w, kc, kcs, cl = d.codes()
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        idx, cand = pv.decode(batch, mode, 128, 32, want_cand=True)
        oidx, ocand, _ = oracle.decode(F32, q, qs, w, kc, kcs, cl, mode, 128, 32)
        assert_rows_exact(idx.cpu().reshape(-1, 32), oidx.reshape(-1, 32), f"decode {mode}")
        if mode != pv.DENSE:
            assert_rows_exact(cand.cpu(), ocand, "decode cand")


# ---------------------------------------------------------------------------
# bounded waits
# ---------------------------------------------------------------------------

def test_bounded_wait_returns_timeout_and_device_stays_usable(tiny):
    p, dev, cfg = tiny
    assert pv.device_error() == 0
    try:
        assert pv.pivot_set_wait_limit_ns(2_000_000) == 0          # 2 ms
        assert pv.pivot_selftest_wait_timeout(None) == 0
        assert pv.device_error() == 5                                # PIVOT_ERR_TIMEOUT
    finally:
        assert pv.pivot_set_wait_limit_ns(0) == 0
    assert pv.device_error() == 0
    idx, _ = pv.dense_index(seq_of(dev), cfg["topk"])               # context still fine
    torch.cuda.synchronize()
    assert idx.shape == (p.L, cfg["topk"])
