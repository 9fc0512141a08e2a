"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
run the library through its C ABI, compare with the oracle.

Comparison rules (the indexer returns positions in rank order):
* integer-valued inputs: every score is exact in fp32 and fp64, so index
  rows must be identical, order and -1 padding included;
* real-valued inputs: GPU scores accumulate in fp32 (tensor cores) while the
  oracle is fp64, so rows may differ only at the selection boundary.  With
  s_k the oracle's k-th score (the lowest selected one; rows list positions
  in ascending order) and tol = 1e-3 * |s_k|: every position the GPU
  picked that the oracle did not must score >= s_k - tol (by the oracle),
  and every position the oracle picked that the GPU did not must score
  <= s_k + tol; GPU scores must be within tol of the oracle's.
"""
import numpy as np
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

REL_TOL = 1e-3


def to_device(p):
    d = "cuda"
    return dict(q=p.q.to(d), q_scale=None if p.q_scale is None else p.q_scale.to(d),
                w=p.w.to(d), k=p.k.to(d), k_scale=None if p.k_scale is None else p.k_scale.to(d))


def seq_of(dev, t_begin=0, t_end=0):
    return pv.make_seq(dev["q"], dev["q_scale"], dev["w"], dev["k"], dev["k_scale"], t_begin,
                       t_end)


def assert_rows_exact(gpu, ref, what=""):
    gpu = np.asarray(gpu)
    ref = np.asarray(ref)
    if not (gpu == ref).all():
        bad = np.nonzero((gpu != ref).any(axis=1))[0]
        r = bad[0]
        raise AssertionError(f"{what}: {len(bad)} rows differ; first row {r}: "
                             f"gpu {gpu[r][:16]} ref {ref[r][:16]}")


def assert_rows_close(gpu_idx, ref_idx, ref_scores, score_fn, rows, what="", gpu_scores=None,
                      abs_tol=None):
    """Boundary-tolerant set comparison, row by row (see module doc).
    `abs_tol(row)`, when given, replaces the relative tolerance by an
    absolute bound derived for that row's arithmetic."""
    gpu_idx = np.asarray(gpu_idx)
    ref_idx = np.asarray(ref_idx)
    nbad = 0
    for i, r in enumerate(rows):
        g = [x for x in gpu_idx[i] if x >= 0]
        o = [x for x in ref_idx[i] if x >= 0]
        assert len(g) == len(o), f"{what} row {r}: gpu picked {len(g)}, oracle {len(o)}"
        if not o:
            continue
        sk = float(np.min(ref_scores[i][:len(o)]))     # the k-th score: rows are listed by position
        tol = REL_TOL * max(abs(sk), 1e-30) if abs_tol is None else abs_tol(r)
        gs, os_ = set(g), set(o)
        only_g = sorted(gs - os_)
        only_o = sorted(os_ - gs)
        if only_g:
            sc = score_fn(r, only_g)
            if (sc < sk - tol).any():
                nbad += 1
                raise AssertionError(f"{what} row {r}: gpu-only positions score below the "
                                     f"boundary {sk}: {list(zip(only_g, sc))[:5]}")
        if only_o:
            refs = dict(zip(o, ref_scores[i][:len(o)]))
            worst = max(refs[x] for x in only_o)
            assert worst <= sk + tol, f"{what} row {r}: oracle-only position scores {worst} > {sk}"
        if gpu_scores is not None:
            gsc = np.asarray(gpu_scores[i][:len(g)], dtype=np.float64)
            want = score_fn(r, g)
            err = np.abs(gsc - want).max()
            assert err <= tol, f"{what} row {r}: score error {err} > {tol}"
    return nbad


def tf32_abs_tol(pq, pw, k):
    """Error bound of one score when the tensor cores consume fp32 operands
    at TF32 (10 explicit mantissa bits; truncation at worst): each product
    q*k is off by at most 2^-9 |q||k| relative, plus fp32 accumulation, so
    |err| <= 2^-8 * sum_h |w_h| sum_d |q_hd| |k_d|.  Returns a per-row bound
    (max over the row's keys)."""
    aq = np.abs(pq.astype(np.float64))                 # [G, H, D]
    ak = np.abs(k.astype(np.float64))                  # [L, D]
    bound = np.einsum("gh,ghd->gd", np.abs(pw.astype(np.float64)), aq) @ ak.T   # [G, L]
    per_row = bound.max(axis=1) * 2.0 ** -8

    def fn(j):
        return per_row[j]
    return fn


def oracle_codes(p):
    return p.codes()


def score_fn_for(p):
    q, qs, w, k, ks = p.codes()

    def fn(row, positions):
        return oracle.score_positions(p.dtype, q, qs, w, k, ks, row, positions)
    return fn


def proxy_score_fn(p, pq, pqs, pw):
    _, _, _, k, ks = p.codes()
    pq = gen.codes_of(pq.cpu(), p.dtype) if isinstance(pq, torch.Tensor) else pq

    def fn(j, positions):
        return oracle.score_positions(p.dtype, pq, pqs, pw, k, ks, j, positions)
    return fn
