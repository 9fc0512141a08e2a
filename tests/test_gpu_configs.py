"""GPU parity at the workloads' own sizes: k = 2048, C = 4096 / 8192, H = 64,
D = 128, the DSA-shaped generator, through the C ABI in the launch
configuration the benchmark times (default workspaces, whole-sequence calls).

Each test names the workload it stands for:
* dsa_prefill_16k: L = 16384, bf16, g = 8, C = 4096;
* fp8_prefill_16k: the same with FP8 e4m3 codes and per-token scales;
* dsa_prefill_64k at g = 16, C = 8192 (the sweep's widest point);
* long_prefill_128k_fp8: L = 131072, FP8, g = 8, C = 4096 (the headline),
  and the same sizes with integer-valued bf16 codes (exact scores, ties);
* mtp_decode_b32: 32 cached sequences of 32768..131072 FP8 keys, two MTP
  tokens per step, C = 4096, k = 2048.

An oracle row at these sizes costs up to ~1e9 fp64 multiply-adds, so each
test checks a sample: rows spread over all positions plus the first and last
rows (dense, Refine) and groups (proxy scan), rows on both sides of k (where
every eligible position is selected) and, for decode, a sample of the
sequences.  Dense and the proxy scan are compared with the oracle's own
rows; Reuse (exactly) and Refine (within tolerance) are compared with the
oracle run on the GPU's candidates, which isolates each step.  Real-valued
rows compare within the boundary tolerance of tests/parity.py.
"""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import (assert_rows_close, assert_rows_exact, proxy_score_fn, score_fn_for, seq_of,
                    to_device)

pytestmark = pytest.mark.gpu

BF16, E4M3 = gen.BF16, gen.E4M3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


def _sample(n, count, extra=()):
    s = set(np.linspace(0, n - 1, count).astype(int)) | {0, n - 1} | set(extra)
    return np.array(sorted(x for x in s if 0 <= x < n))


def _check_prefill(p, g, C, kk, nrows=24, ngroups=16):
    L = p.L
    dev = to_device(p)
    seq = seq_of(dev)
    q, qs, w, k, ks = p.codes()
    rows = _sample(L, nrows, extra=(kk - 2, kk - 1, kk, kk + 1, C - 1, C))
    G = -(-L // g)
    groups = _sample(G, ngroups, extra=((C // g) - 1, C // g))

    # dense
    idx, sc = pv.dense_index(seq, kk, with_score=True)
    gi, gs = idx[rows].cpu().numpy(), sc[rows].cpu().numpy()
    del idx, sc
    oidx, osc = oracle.dense_index(p.dtype, q, qs, w, k, ks, kk, rows=rows)
    fn = score_fn_for(p)
    assert_rows_close(gi, oidx, osc, fn, rows, "dense", gpu_scores=gs)

    # PIVOT: proxy reduce (bit for bit), proxy scan, Reuse, Refine
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
    reu = pv.reuse(0, L, g, cand, kk)
    ref, rs = pv.refine(seq, g, cand, kk, with_score=True)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    opq, opqs, opw = oracle.proxy_reduce(p.dtype, q, qs, w, g)
    assert (gen.codes_of(pq.cpu(), p.dtype) == opq).all()
    assert (pw.cpu().numpy() == opw).all()
    if p.dtype == E4M3:
        assert (pqs.cpu().numpy() == opqs).all()
    gc_s, gcs_s = cand[groups].cpu().numpy(), cs[groups].cpu().numpy()
    ocand, ocs = oracle.proxy_scan(p.dtype, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
    pfn = proxy_score_fn(p, opq, opqs, opw)
    assert_rows_close(gc_s, ocand, ocs, pfn, groups, "cand", gpu_scores=gcs_s)
    # the first k entries of a candidate row are the proxy's own top-k
    assert_rows_close(gc_s[:, :kk], ocand[:, :kk], ocs[:, :kk], pfn, groups, "cand top-k",
                      gpu_scores=gcs_s[:, :kk])

    gcand = cand.cpu().numpy()
    assert_rows_exact(reu[rows].cpu().numpy(), oracle.reuse(L, g, gcand, kk, rows=rows), "reuse")
    oref, ors = oracle.refine(p.dtype, q, qs, w, k, ks, g, gcand, kk, rows=rows)
    assert_rows_close(ref[rows].cpu().numpy(), oref, ors, fn, rows, "refine",
                      gpu_scores=rs[rows].cpu().numpy())


def _workload(name, **over):
    cfg = dict(gen.WORKLOADS[name])
    cfg.update(over)
    p = gen.make_prefill(cfg["L"], cfg["H"], cfg["D"], cfg["dtype"], kind=cfg["kind"], seed=0)
    return p, cfg


def test_dsa_prefill_16k_bf16():
    p, cfg = _workload("dsa_prefill_16k")
    _check_prefill(p, cfg["g"], cfg["C"], cfg["topk"])


def test_fp8_prefill_16k():
    p, cfg = _workload("fp8_prefill_16k")
    _check_prefill(p, cfg["g"], cfg["C"], cfg["topk"])


def test_dsa_prefill_64k_g16_c8192():
    p, cfg = _workload("dsa_prefill_64k")
    _check_prefill(p, 16, 8192, cfg["topk"], nrows=16, ngroups=12)


def test_long_prefill_128k_fp8_sampled():
    p, cfg = _workload("long_prefill_128k_fp8")
    _check_prefill(p, cfg["g"], cfg["C"], cfg["topk"], nrows=16, ngroups=12)


def test_long_prefill_128k_integer_exact():
    """Integer-valued bf16 codes at the headline's sizes (L = 131072, H = 64,
    D = 128, g = 8, C = 4096, k = 2048): every score is exact in fp32 and
    equal scores are common, so sampled dense rows, candidate rows (the
    proxy's top-k first), Reuse and Refine rows equal the oracle's bit for
    bit -- the long rows' selection in two CTAs an SM, and its search among
    tied scores, included."""
    L, g, C, kk = 131072, 8, 4096, 2048
    p = gen.make_prefill(L, 64, 128, BF16, kind="int", seed=9)
    dev = to_device(p)
    seq = seq_of(dev)
    q, qs, w, k, ks = p.codes()
    rows = _sample(L, 12, extra=(kk - 1, kk, C))
    groups = _sample(L // g, 10, extra=(C // g - 1, C // g))
    idx, _ = pv.dense_index(seq, kk)
    got = idx[rows].cpu().numpy()
    del idx
    assert_rows_exact(got, oracle.dense_index(BF16, q, qs, w, k, ks, kk, rows=rows)[0], "dense")
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, _ = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)
    reu = pv.reuse(0, L, g, cand, kk)
    ref, _ = pv.refine(seq, g, cand, kk)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    opq, opqs, opw = oracle.proxy_reduce(BF16, q, qs, w, g)
    ocand, _ = oracle.proxy_scan(BF16, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
    assert_rows_exact(cand[groups].cpu().numpy(), ocand, "cand")
    gc = cand.cpu().numpy()
    assert_rows_exact(reu[rows].cpu().numpy(), oracle.reuse(L, g, gc, kk, rows=rows), "reuse")
    assert_rows_exact(ref[rows].cpu().numpy(),
                      oracle.refine(BF16, q, qs, w, k, ks, g, gc, kk, rows=rows)[0], "refine")


def test_mtp_decode_b32_sampled():
    cfg = gen.WORKLOADS["mtp_decode_b32"]
    d = gen.make_decode(B=cfg["B"], Gm=cfg["Gm"], H=cfg["H"], D=cfg["D"], dtype=cfg["dtype"],
                        len_lo=cfg["len_lo"], len_hi=cfg["len_hi"], seed=0)
    c = "cuda"
    batch = pv.make_decode(d.q.to(c), d.q_scale.to(c), d.w.to(c), d.kc.to(c), d.kc_scale.to(c),
                           d.cache_len.to(c))
    C, kk, Gm, dt = cfg["C"], cfg["topk"], cfg["Gm"], cfg["dtype"]
    q, qs, w, kc, kcs, cl = d.codes()
    # the shortest and longest caches and a spread between them
    order = np.argsort(cl)
    bs = sorted({int(order[0]), int(order[-1])} | {int(order[i]) for i in (8, 16, 24)})
    sub = (q[bs], qs[bs], w[bs], kc[bs], kcs[bs], cl[bs])
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        idx, cand = pv.decode(batch, mode, C, kk, want_cand=True)
        torch.cuda.synchronize()
        assert pv.device_error() == 0
        gi = idx.cpu().numpy()[bs]
        oidx, ocand, osc = oracle.decode(dt, *sub, mode, C, kk)
        for i, b in enumerate(bs):
            kb, kbs = kc[b], kcs[b]

            def fn(m, positions, b=b, kb=kb, kbs=kbs):
                return oracle.score_positions(dt, q[b], qs[b], w[b], kb, kbs, m, positions)
            if mode == pv.DENSE:
                assert_rows_close(gi[i], oidx[i], osc[i], fn, list(range(Gm)), f"dense b={b}")
                continue
            gc = cand.cpu().numpy()[b]
            # candidates against the oracle's proxy scan (proxy scores)
            pq, pqs, pw = oracle.proxy_reduce(dt, q[b], qs[b], w[b], Gm)
            n = int(cl[b])

            def pfn(_, positions, kb=kb, kbs=kbs, pq=pq, pqs=pqs, pw=pw):
                return oracle.score_positions(dt, pq, pqs, pw, kb, kbs, 0, positions)
            ocs_b = pfn(0, ocand[i][ocand[i] >= 0])
            assert_rows_close(gc[None, :], ocand[i][None, :], ocs_b[None, :], pfn, [0],
                              f"decode cand b={b}")
            for m in range(Gm):
                lim = n - Gm + m
                if mode == pv.REUSE:
                    want = [x for x in gc[:kk] if 0 <= x <= lim]
                    want += [-1] * (kk - len(want))
                    assert list(gi[i][m]) == want, f"reuse b={b} m={m}"
                else:
                    pos = np.array([x for x in gc if 0 <= x <= lim], dtype=np.int32)
                    sc = fn(m, pos)
                    top = np.lexsort((pos, -sc))[:kk]
                    want = np.array([list(pos[top]) + [-1] * (kk - len(top))])
                    want_sc = np.array([list(sc[top])])
                    assert_rows_close(gi[i][m:m + 1], want, want_sc, fn, [m], f"refine b={b}")
