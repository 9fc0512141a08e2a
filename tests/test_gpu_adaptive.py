"""PIVOT-Refine with a per-group adaptive candidate count (a design choice
of this library; the pages fix C): group j re-scores its first C_j
rank-ordered candidates, those whose proxy score is at least rho times the
proxy's k-th, clamped to [min(k, valid), C]."""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import assert_rows_close, assert_rows_exact, score_fn_for, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


def _seqs(dev):
    args = (dev["q"], dev["q_scale"], dev["w"], dev["k"], dev["k_scale"])
    return (pv.make_seq(*args, order=pv.ORDER_RANK), pv.make_seq(*args))


def expected_counts(cs, kk, rho):
    """The rule in numpy float32 (the product rounded as the kernel rounds it)."""
    out = []
    for row in np.asarray(cs, dtype=np.float32):
        valid = int(np.isfinite(row).sum())
        k = min(kk, valid)
        n = row.shape[0]
        if k > 0 and row[k - 1] > 0:
            T = np.float32(rho) * row[k - 1]
            n = k + int((row[k:valid] >= T).sum())
        out.append(max(n, k))
    return np.array(out)


@pytest.mark.parametrize("rho", [0.0, 0.5, 0.9])
def test_adaptive_refine_integer_exact(rho):
    L, g, C, kk = 5000, 8, 1024, 128
    p = gen.make_prefill(L, 64, 128, gen.BF16, kind="int", seed=12)
    dev = to_device(p)
    rank_seq, pos_seq = _seqs(dev)
    pq, pqs, pw = pv.proxy_reduce(rank_seq, g)
    cand, cs = pv.proxy_scan(rank_seq, g, pq, pqs, pw, C, kk, with_score=True)
    idx, counts = pv.refine_adaptive(pos_seq, g, cand, cs, kk, rho)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    want_counts = expected_counts(cs.cpu().numpy(), kk, rho)
    assert (counts.cpu().numpy() == want_counts).all()
    assert (want_counts >= np.minimum(kk, np.isfinite(cs.cpu().numpy()).sum(1))).all()
    if rho == 0.0:
        plain, _ = pv.refine(pos_seq, g, cand, kk)
        assert torch.equal(idx, plain)
    # the oracle's Refine over each group's first C_j candidates
    gc = cand.cpu().numpy().copy()
    for j, n in enumerate(want_counts):
        gc[j, n:] = -1
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 48).astype(int)) | {L - 1}))
    oref, _ = oracle.refine(gen.BF16, q, qs, w, k, ks, g, gc, kk, rows=rows)
    assert_rows_exact(idx.cpu().numpy()[rows], oref, f"adaptive refine rho={rho}")


def test_adaptive_refine_fp8_fewer_candidates_within_tolerance():
    L, g, C, kk = 16384, 8, 4096, 2048
    p = gen.make_prefill(L, 64, 128, gen.E4M3, kind="dsa", seed=0)
    dev = to_device(p)
    rank_seq, pos_seq = _seqs(dev)
    pq, pqs, pw = pv.proxy_reduce(rank_seq, g)
    cand, cs = pv.proxy_scan(rank_seq, g, pq, pqs, pw, C, kk, with_score=True)
    idx, counts = pv.refine_adaptive(pos_seq, g, cand, cs, kk, 0.8)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    cnt = counts.cpu().numpy()
    assert (cnt == expected_counts(cs.cpu().numpy(), kk, 0.8)).all()
    assert cnt.mean() < C                       # the rule does cut candidates here
    gc = cand.cpu().numpy().copy()
    for j, n in enumerate(cnt):
        gc[j, n:] = -1
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 24).astype(int)) | {L - 1}))
    oref, ors = oracle.refine(gen.E4M3, q, qs, w, k, ks, g, gc, kk, rows=rows)
    assert_rows_close(idx.cpu().numpy()[rows], oref, ors, score_fn_for(p), rows, "adaptive refine")
