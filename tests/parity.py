"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
run the library through its C ABI, compare with the oracle.

Comparison rules (index rows list the selected positions in ascending
order unless rank order is asked for):
* integer-valued inputs: every score is exact in fp32 and fp64, so index
  rows must be identical, order and -1 padding included;
* real-valued inputs: GPU scores accumulate in fp32 (tensor cores) while the
  oracle is fp64, so rows may differ only at the selection boundary.  With
  s_k the oracle's k-th score (the lowest selected one) and
  tol = 1e-3 * |s_k|: every position the GPU picked that the oracle did
  not must score >= s_k - tol (by the oracle), and every position the
  oracle picked that the GPU did not must score <= s_k + tol; each GPU
  score s must be within max(1e-3 * |s_ref|, tol) of the oracle's s_ref.
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
    `abs_tol(row)`, when given, is a floor on every tolerance of that row:
    the error bound of its fp32 arithmetic (fp32_abs_tol)."""
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
        tol = REL_TOL * max(abs(sk), 1e-30)
        if abs_tol is not None:
            tol = max(tol, abs_tol(r))
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
            # each score within 1e-3 of itself, and never held tighter than
            # the boundary's tolerance (a row whose k-th score is 0 -- ReLU
            # zeros -- still compares its other scores relatively)
            gsc = np.asarray(gpu_scores[i][:len(g)], dtype=np.float64)
            want = score_fn(r, g)
            stol = np.maximum(REL_TOL * np.abs(want), tol)
            bad = np.abs(gsc - want) > stol
            assert not bad.any(), (f"{what} row {r}: score error "
                                   f"{np.abs(gsc - want)[bad].max()} > {stol[bad].min()}")
    return nbad


def fp32_abs_tol(pq, pw, k):
    """The error bound of a score computed in fp32 on the CUDA cores (each
    head's dot product a chain of D fused multiply-adds, then a chain of H
    weighted adds): |err| <= (D + H + 2) u sum_h |w_h| sum_d |q_hd| |k_d|,
    u = 2^-24 (the standard bound on recursive summation, Higham, Accuracy
    and Stability of Numerical Algorithms, ch. 3), taken twice for margin.
    It matters where a row's boundary sits among near-zero scores that come
    from cancelling dot products, which no relative tolerance can scale.
    Returns a per-row bound (max over the row's keys)."""
    pq = np.asarray(pq, dtype=np.float64)
    H, D = pq.shape[1], pq.shape[2]
    bound = np.einsum("gh,ghd->gd", np.abs(np.asarray(pw, dtype=np.float64)), np.abs(pq)) @ \
        np.abs(np.asarray(k, dtype=np.float64)).T
    per_row = bound.max(axis=1) * 2.0 * (D + H + 2) * 2.0 ** -24

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
