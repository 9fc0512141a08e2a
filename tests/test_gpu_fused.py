"""The selection fused into the scan (dense and proxy rows on the tensor
cores): a sample scan bounds each row, the scan keeps only the scores at or
above the bound, one warp per row selects among them, and rows whose
survivors fall outside that range are rescanned keeping everything.

* The fused path and the path that writes every score compute the same fp32
  scores, so their index rows must be identical, order and padding included.
* Forcing every long row through the rescan (the bound far too high, or far
  too low) must change nothing.
* Integer-valued bf16 inputs at H = 64, D = 128 make every score exact and
  heavily tied: the fused rows must equal the oracle's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import assert_rows_exact, seq_of, to_device

pytestmark = pytest.mark.gpu

BF16, E4M3 = gen.BF16, gen.E4M3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()
    yield
    pv.pivot_set_fused_selection(0, 4.5)   # the default


def _dense_and_cand(dev, L, g, C, kk, order=pv.ORDER_POSITION):
    seq = pv.make_seq(dev["q"], dev["q_scale"], dev["w"], dev["k"], dev["k_scale"], order=order)
    idx, sc = pv.dense_index(seq, kk, with_score=True)
    pq, pqs, pw = pv.proxy_reduce(seq, g)
    cand, cs = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk, with_score=True)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    return idx, sc, cand, cs


@pytest.mark.parametrize("dtype,L,kk,C", [(E4M3, 16384, 2048, 4096), (BF16, 9000, 300, 2600),
                                          (E4M3, 5000, 2048, 8192)])
def test_fused_equals_writing_every_score(dtype, L, kk, C):
    p = gen.make_prefill(L, 64, 128, dtype, kind="dsa", seed=21)
    dev = to_device(p)
    g = 8
    try:
        assert pv.pivot_set_fused_selection(0, 4.5) == 0
        ref = _dense_and_cand(dev, L, g, C, kk)
        assert pv.pivot_set_fused_selection(1, 4.5) == 0
        got = _dense_and_cand(dev, L, g, C, kk)
        for a, b, what in zip(got, ref, ("dense", "dense scores", "cand", "cand scores")):
            assert torch.equal(a, b), what
        # both ways through the rescan: bound far too high, far too low
        for sig in (-60.0, 600.0):
            assert pv.pivot_set_fused_selection(1, sig) == 0
            got = _dense_and_cand(dev, L, g, C, kk)
            for a, b, what in zip(got, ref, ("dense", "dense scores", "cand", "cand scores")):
                assert torch.equal(a, b), (what, sig)
        # rank order too
        assert pv.pivot_set_fused_selection(0, 4.5) == 0
        ref_r = _dense_and_cand(dev, L, g, C, kk, pv.ORDER_RANK)
        assert pv.pivot_set_fused_selection(1, 4.5) == 0
        got_r = _dense_and_cand(dev, L, g, C, kk, pv.ORDER_RANK)
        for a, b, what in zip(got_r, ref_r, ("dense", "dense scores", "cand", "cand scores")):
            assert torch.equal(a, b), ("rank", what)
    finally:
        pv.pivot_set_fused_selection(0, 4.5)


@pytest.mark.parametrize("sig", [4.5, -60.0])
def test_fused_integer_rows_exact(sig):
    """Small integers in bf16 at H = 64, D = 128: exact fp32 scores with many
    ties; dense, candidates, Reuse and Refine equal the oracle's rows."""
    L, g, C, kk = 6000, 8, 1024, 256
    p = gen.make_prefill(L, 64, 128, BF16, kind="int", seed=5)
    dev = to_device(p)
    q, qs, w, k, ks = p.codes()
    rows = np.array(sorted(set(np.linspace(0, L - 1, 40).astype(int)) | {kk - 1, kk, L - 1}))
    groups = np.array(sorted(set(np.linspace(0, L // g - 1, 24).astype(int))))
    try:
        assert pv.pivot_set_fused_selection(1, sig) == 0
        seq = seq_of(dev)
        idx, sc = pv.dense_index(seq, kk, with_score=True)
        oidx, osc = oracle.dense_index(BF16, q, qs, w, k, ks, kk, rows=rows)
        assert_rows_exact(idx.cpu().numpy()[rows], oidx, "dense")
        ok = oidx >= 0
        assert (sc.cpu().numpy()[rows][ok] == osc[ok]).all()
        pq, pqs, pw = pv.proxy_reduce(seq, g)
        cand, _ = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)
        opq, opqs, opw = oracle.proxy_reduce(BF16, q, qs, w, g)
        ocand, _ = oracle.proxy_scan(BF16, opq, opqs, opw, k, ks, L, g, C, kk, groups=groups)
        assert_rows_exact(cand.cpu().numpy()[groups], ocand, "cand")
        reu = pv.reuse(0, L, g, cand, kk)
        ref, _ = pv.refine(seq, g, cand, kk)
        torch.cuda.synchronize()
        assert pv.device_error() == 0
        gc = cand.cpu().numpy()
        assert_rows_exact(reu.cpu().numpy()[rows], oracle.reuse(L, g, gc, kk, rows=rows), "reuse")
        assert_rows_exact(ref.cpu().numpy()[rows],
                          oracle.refine(BF16, q, qs, w, k, ks, g, gc, kk, rows=rows)[0], "refine")
    finally:
        pv.pivot_set_fused_selection(0, 4.5)


def test_fused_row_ranges_and_small_workspace():
    """Row ranges (as ranks split a sequence) and a workspace that forces
    many launches give the single call's rows."""
    L, kk = 7000, 512
    p = gen.make_prefill(L, 64, 128, E4M3, kind="dsa", seed=3)
    dev = to_device(p)
    assert pv.pivot_set_fused_selection(1, 4.5) == 0
    full, _ = pv.dense_index(seq_of(dev), kk)
    a, _ = pv.dense_index(seq_of(dev, 0, 3000), kk)
    b, _ = pv.dense_index(seq_of(dev, 3000, L), kk)
    assert torch.equal(torch.cat([a, b]), full)
    need = pv.pivot_dense_index_workspace_size(seq_of(dev), kk)
    small = torch.empty(need // 9, dtype=torch.uint8, device="cuda")
    c, _ = pv.dense_index(seq_of(dev), kk, ws=small)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    assert torch.equal(c, full)
    assert pv.pivot_set_fused_selection(0, 4.5) == 0
    assert torch.equal(pv.dense_index(seq_of(dev), kk)[0], full)


@pytest.mark.parametrize("dtype,Gm", [(E4M3, 2), (BF16, 3)])
def test_fused_decode_equals_writing_every_score(dtype, Gm):
    """MTP decode over ragged cache lengths: dense and
    proxy rows through the fused selection equal the rows written from every
    score, in both output orders and through the forced rescan."""
    d = gen.make_decode(B=6, Gm=Gm, H=64, D=128, dtype=dtype, len_lo=3000, len_hi=20000, seed=17)
    c = "cuda"
    C, kk = 4096, 2048
    try:
        for order in (pv.ORDER_POSITION, pv.ORDER_RANK):
            batch = pv.make_decode(d.q.to(c), None if d.q_scale is None else d.q_scale.to(c),
                                   d.w.to(c), d.kc.to(c),
                                   None if d.kc_scale is None else d.kc_scale.to(c),
                                   d.cache_len.to(c), order=order)
            want = {}
            assert pv.pivot_set_fused_selection(0, 4.5) == 0
            for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
                want[mode] = pv.decode(batch, mode, C, kk, want_cand=True)
            for sig in (4.5, -60.0, 600.0):
                assert pv.pivot_set_fused_selection(1, sig) == 0
                for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
                    idx, cand = pv.decode(batch, mode, C, kk, want_cand=True)
                    torch.cuda.synchronize()
                    assert pv.device_error() == 0
                    assert torch.equal(idx, want[mode][0]), (order, sig, mode)
                    if mode != pv.DENSE:
                        assert torch.equal(cand, want[mode][1]), (order, sig, mode)
    finally:
        pv.pivot_set_fused_selection(0, 4.5)
