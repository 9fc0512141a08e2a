"""CPU oracle for the PIVOT indexer -- test infrastructure, not the product.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product library never links or calls it,
and this package imports nothing from the product: the two share no code.

The arithmetic lives in ``pivot_oracle.c`` (plain C, fp64 scores, fp32 proxy
without FMA contraction); this module only builds it with gcc and marshals
numpy arrays through ctypes.  Every function cites the page it follows in the
C source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pivot_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, E4M3 = 0, 1, 2
DENSE, REUSE, REFINE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, no FMA contraction)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_e4m3_to_double.restype = ctypes.c_double
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_double_to_e4m3_satfinite.restype = ctypes.c_uint8
            lib.oracle_double_to_e4m3_satfinite.argtypes = [ctypes.c_double]
            lib.oracle_bf16_to_double.restype = ctypes.c_double
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_float_to_bf16_rne.restype = ctypes.c_uint16
            lib.oracle_float_to_bf16_rne.argtypes = [ctypes.c_float]
            lib.oracle_max_threads.restype = I
            lib.oracle_score_positions.argtypes = [I, I, I, I, P, P, P, P, P, I, I, P, P]
            lib.oracle_dense_index.argtypes = [I, I, I, I, P, P, P, P, P, I, I, P, P, P, I]
            lib.oracle_proxy_reduce.argtypes = [I, I, I, I, P, P, P, I, I, P, P, P, P]
            lib.oracle_proxy_scan.argtypes = [I, I, I, I, P, P, P, P, P, I, I, I, I, P, P, P, I]
            lib.oracle_reuse.argtypes = [I, I, P, I, I, I, P, P]
            lib.oracle_refine.argtypes = [I, I, I, I, P, P, P, P, P, I, P, I, I, I, P, P, P, I]
            lib.oracle_decode.argtypes = [I, I, I, I, I, P, P, P, P, P, I, P, I, I, I, P, P, P, I]
            lib.oracle_window_union.argtypes = [P, I, I, I, P]
            lib.oracle_reuse_backfill.argtypes = [I, I, P, P, I, I, I, P, P]
            _lib = lib
    return _lib


# --------------------------------------------------------------------------
# marshalling helpers
# --------------------------------------------------------------------------

def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _codes(x, dtype):
    """Raw storage of an input: float32 array, uint16 bf16 codes or uint8 e4m3 codes."""
    want = {F32: np.float32, BF16: np.uint16, E4M3: np.uint8}[dtype]
    x = np.ascontiguousarray(x)
    assert x.dtype == want, f"dtype code {dtype} needs {want}, got {x.dtype}"
    return x


def _f32(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float32)


def _rows(rows, n):
    if rows is None:
        rows = np.arange(n, dtype=np.int32)
    return np.ascontiguousarray(rows, dtype=np.int32)


def max_threads() -> int:
    return int(_load().oracle_max_threads())


# --------------------------------------------------------------------------
# formats
# --------------------------------------------------------------------------

def e4m3_to_float(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint8).ravel()
    out = np.array([lib.oracle_e4m3_to_double(int(c)) for c in flat], dtype=np.float64)
    return out.reshape(np.shape(codes))


def float_to_e4m3(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float64).ravel()
    out = np.array([lib.oracle_double_to_e4m3_satfinite(float(v)) for v in flat], dtype=np.uint8)
    return out.reshape(np.shape(x))


def bf16_to_float(codes: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(codes, dtype=np.uint16).ravel()
    out = np.array([lib.oracle_bf16_to_double(int(c)) for c in flat], dtype=np.float64)
    return out.reshape(np.shape(codes))


def float_to_bf16(x: np.ndarray) -> np.ndarray:
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).ravel()
    out = np.array([lib.oracle_float_to_bf16_rne(float(v)) for v in flat], dtype=np.uint16)
    return out.reshape(np.shape(x))


# --------------------------------------------------------------------------
# the method
# --------------------------------------------------------------------------

def score_positions(dtype, q, q_scale, w, k, k_scale, row, positions):
    """I(row, s) for each listed s (fp64), no selection."""
    lib = _load()
    _, H, D = q.shape
    nkeys = k.shape[0]
    q, k = _codes(q, dtype), _codes(k, dtype)
    q_scale, k_scale, w = _f32(q_scale), _f32(k_scale), _f32(w)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    out = np.zeros(len(pos), dtype=np.float64)
    lib.oracle_score_positions(dtype, nkeys, H, D, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k),
                               _ptr(k_scale), int(row), len(pos), _ptr(pos), _ptr(out))
    return out


def dense_index(dtype, q, q_scale, w, k, k_scale, topk, rows=None, nthreads=0):
    """Dense indexer: top-k positions, ascending (and their fp64 scores), of
    each listed row."""
    lib = _load()
    L, H, D = q.shape
    q, k = _codes(q, dtype), _codes(k, dtype)
    q_scale, k_scale, w = _f32(q_scale), _f32(k_scale), _f32(w)
    rows = _rows(rows, L)
    idx = np.empty((len(rows), topk), dtype=np.int32)
    sc = np.empty((len(rows), topk), dtype=np.float64)
    lib.oracle_dense_index(dtype, L, H, D, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k),
                           _ptr(k_scale), topk, len(rows), _ptr(rows), _ptr(idx), _ptr(sc),
                           nthreads)
    return idx, sc


def proxy_reduce(dtype, q, q_scale, w, g, groups=None):
    """Proxy query, scale and weights of each listed prefill group."""
    lib = _load()
    L, H, D = q.shape
    G = (L + g - 1) // g
    q = _codes(q, dtype)
    q_scale, w = _f32(q_scale), _f32(w)
    groups = _rows(groups, G)
    store = {F32: np.float32, BF16: np.uint16, E4M3: np.uint8}[dtype]
    pq = np.zeros((len(groups), H, D), dtype=store)
    pqs = np.ones(len(groups), dtype=np.float32) if dtype == E4M3 else None
    pw = np.zeros((len(groups), H), dtype=np.float32)
    lib.oracle_proxy_reduce(dtype, L, H, D, _ptr(q), _ptr(q_scale), _ptr(w), g, len(groups),
                            _ptr(groups), _ptr(pq), _ptr(pqs), _ptr(pw))
    return pq, pqs, pw


def proxy_scan(dtype, pq, pq_scale, pw, k, k_scale, L, g, C, topk, groups=None, nthreads=0):
    """Top-C candidates of each listed group's proxy over [0, e_j]: the
    top-`topk` positions ascending, then the rest ascending."""
    lib = _load()
    G, H, D = pq.shape
    pq, k = _codes(pq, dtype), _codes(k, dtype)
    pq_scale, pw, k_scale = _f32(pq_scale), _f32(pw), _f32(k_scale)
    groups = _rows(groups, G)
    cand = np.empty((len(groups), C), dtype=np.int32)
    sc = np.empty((len(groups), C), dtype=np.float64)
    lib.oracle_proxy_scan(dtype, L, H, D, _ptr(pq), _ptr(pq_scale), _ptr(pw), _ptr(k),
                          _ptr(k_scale), g, C, topk, len(groups), _ptr(groups), _ptr(cand),
                          _ptr(sc), nthreads)
    return cand, sc


def reuse(L, g, cand, topk, rows=None):
    """PIVOT-Reuse rows from the full candidate table cand [G, C]."""
    lib = _load()
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    G, C = cand.shape
    rows = _rows(rows, L)
    out = np.empty((len(rows), topk), dtype=np.int32)
    lib.oracle_reuse(L, g, _ptr(cand), C, topk, len(rows), _ptr(rows), _ptr(out))
    return out


def reuse_backfill(L, g, cand, cand_score, topk, rows=None):
    """Reuse with backfill: per member, the top-k of its group's candidates at
    positions <= t by proxy score (cand_score, same shape as cand)."""
    lib = _load()
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    cand_score = np.ascontiguousarray(cand_score, dtype=np.float64)
    assert cand_score.shape == cand.shape
    G, C = cand.shape
    rows = _rows(rows, L)
    out = np.empty((len(rows), topk), dtype=np.int32)
    lib.oracle_reuse_backfill(L, g, _ptr(cand), _ptr(cand_score), C, topk, len(rows), _ptr(rows),
                              _ptr(out))
    return out


def index_window_outside(dtype, q, q_scale, w, k, k_scale, mode, g, C, topk, window, rows=None):
    """The window kept out of the candidates: row t chooses by `mode` (DENSE,
    REUSE, REFINE) among positions <= t - window only, then the window
    [t - window + 1, t] is added.  [rows, topk + window], ascending, -1 padded.
    Built from the functions above, row by row (small inputs only)."""
    L = q.shape[0]
    rows = _rows(rows, L)
    out = np.full((len(rows), topk + window), -1, dtype=np.int32)
    if mode != DENSE:
        pq, pqs, pw = proxy_reduce(dtype, q, q_scale, w, g)
        cand, _ = proxy_scan(dtype, pq, pqs, pw, k, k_scale, L, g, C, topk)
    for r, t in enumerate(rows):
        lim = t - window
        if mode == REUSE:
            sel = [s for s in cand[t // g, :topk] if 0 <= s <= lim]
        else:
            if mode == DENSE:
                pos = np.arange(0, lim + 1, dtype=np.int32)
            else:
                pos = np.array([s for s in cand[t // g] if 0 <= s <= lim], dtype=np.int32)
            sel = []
            if len(pos):
                sc = score_positions(dtype, q, q_scale, w, k, k_scale, t, pos)
                order = np.lexsort((pos, -sc))[:topk]
                sel = sorted(pos[order].tolist())
        u = window_union(np.array(sel, dtype=np.int32), int(t), window)
        out[r, :len(u)] = u
    return out


def window_union_rows(idx, t_first, window):
    """Each index row (ascending, -1 padded) united with its window
    [t - window + 1, t], t = t_first + row: [rows, k + window], -1 padded."""
    idx = np.asarray(idx, dtype=np.int32)
    rows, k = idx.shape
    out = np.full((rows, k + window), -1, dtype=np.int32)
    for r in range(rows):
        sel = idx[r][idx[r] >= 0]
        u = window_union(sel, t_first + r, window)
        out[r, :len(u)] = u
    return out


def refine(dtype, q, q_scale, w, k, k_scale, g, cand, topk, rows=None, nthreads=0):
    """PIVOT-Refine rows from the full candidate table cand [G, C]."""
    lib = _load()
    L, H, D = q.shape
    q, k = _codes(q, dtype), _codes(k, dtype)
    q_scale, k_scale, w = _f32(q_scale), _f32(k_scale), _f32(w)
    cand = np.ascontiguousarray(cand, dtype=np.int32)
    C = cand.shape[1]
    rows = _rows(rows, L)
    idx = np.empty((len(rows), topk), dtype=np.int32)
    sc = np.empty((len(rows), topk), dtype=np.float64)
    lib.oracle_refine(dtype, L, H, D, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(k), _ptr(k_scale),
                      g, _ptr(cand), C, topk, len(rows), _ptr(rows), _ptr(idx), _ptr(sc),
                      nthreads)
    return idx, sc


def decode(dtype, q, q_scale, w, kc, kc_scale, cache_len, mode, C, topk, nthreads=0):
    """One MTP decode step for a batch; returns (idx [B,Gm,k], cand [B,C] or None, scores)."""
    lib = _load()
    B, Gm, H, D = q.shape
    maxlen = kc.shape[1]
    q, kc = _codes(q, dtype), _codes(kc, dtype)
    q_scale, kc_scale, w = _f32(q_scale), _f32(kc_scale), _f32(w)
    cl = np.ascontiguousarray(cache_len, dtype=np.int32)
    idx = np.empty((B, Gm, topk), dtype=np.int32)
    cand = np.empty((B, C), dtype=np.int32) if mode != DENSE else None
    sc = np.empty((B, Gm, topk), dtype=np.float64)
    lib.oracle_decode(dtype, B, Gm, H, D, _ptr(q), _ptr(q_scale), _ptr(w), _ptr(kc),
                      _ptr(kc_scale), maxlen, _ptr(cl), mode, C, topk, _ptr(idx), _ptr(cand),
                      _ptr(sc), nthreads)
    return idx, cand, sc


def window_union(selected, t, window):
    """Selected positions united with the recent window [t-window+1, t], ascending."""
    lib = _load()
    sel = np.ascontiguousarray(selected, dtype=np.int32)
    out = np.empty(t + 1, dtype=np.int32)
    n = lib.oracle_window_union(_ptr(sel), len(sel), int(t), int(window), _ptr(out))
    return out[:n]
