"""Python binding of libpivot (ctypes).

The functions named ``pivot_*`` mirror the C ABI of ``include/pivot.h`` one
to one (argument marshalling only).  The lower-case helpers below them
(``dense_index``, ``proxy_reduce``, ...) allocate outputs and workspaces
with torch on the caller's device and stream and then call the same entry
points; every step of the indexer runs in the library's CUDA kernels.

There is no fallback: if ``libpivot.so`` is missing or cannot be loaded,
``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpivot.so")

F32, BF16, E4M3 = 0, 1, 2
DENSE, REUSE, REFINE = 0, 1, 2
ORDER_POSITION, ORDER_RANK = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace too small",
          4: "CUDA error", 5: "a kernel wait timed out", 6: "bad device-side data"}

ABI_SYMBOLS = [
    "pivot_dense_index", "pivot_dense_index_workspace_size", "pivot_proxy_reduce",
    "pivot_proxy_scan", "pivot_proxy_scan_workspace_size", "pivot_reuse", "pivot_refine",
    "pivot_refine_workspace_size", "pivot_decode", "pivot_decode_workspace_size",
    "pivot_get_device_error", "pivot_set_wait_limit_ns", "pivot_selftest_wait_timeout",
    "pivot_status_string", "pivot_version", "pivot_profile_enable", "pivot_profile_read",
    "pivot_launch_count", "pivot_decode_noalloc", "pivot_last_error_detail",
    "pivot_reuse_backfill", "pivot_window_union", "pivot_index_varlen",
    "pivot_index_varlen_workspace_size", "pivot_index_window_outside",
    "pivot_index_window_outside_workspace_size", "pivot_set_score_buffer_cap",
    "pivot_workspace_size", "pivot_set_fused_selection", "pivot_refine_adaptive",
    "pivot_refine_adaptive_workspace_size",
]
KERNELS = {0: "scan", 1: "select", 2: "refine", 3: "reduce", 4: "reuse"}


class PivotError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} (status {status})")


class PivotSeq(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("L", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p),
                ("w", ctypes.c_void_p), ("k", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("t_begin", ctypes.c_int32), ("t_end", ctypes.c_int32),
                ("order", ctypes.c_int32)]


class PivotVarlen(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("nseq", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p), ("q", ctypes.c_void_p),
                ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("order", ctypes.c_int32)]


class PivotDecode(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("B", ctypes.c_int32), ("Gm", ctypes.c_int32),
                ("H", ctypes.c_int32), ("D", ctypes.c_int32), ("maxlen", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("q_scale", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("kc", ctypes.c_void_p), ("kc_scale", ctypes.c_void_p),
                ("cache_len", ctypes.c_void_p), ("order", ctypes.c_int32)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libpivot.so (raises if it is missing: there is no other path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libpivot.so not built at {path}; run "
                          "`python -m top_token_selection_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    sig = {
        "pivot_dense_index": ([P, I32, P, P, P, SZ, P], I32),
        "pivot_dense_index_workspace_size": ([P, I32], SZ),
        "pivot_proxy_reduce": ([P, I32, P, P, P, P], I32),
        "pivot_proxy_scan": ([P, I32, P, P, P, I32, I32, P, P, P, SZ, P], I32),
        "pivot_proxy_scan_workspace_size": ([P, I32, I32], SZ),
        "pivot_reuse": ([I32, I32, I32, P, I32, I32, P, P], I32),
        "pivot_refine": ([P, I32, P, I32, I32, P, P, P, SZ, P], I32),
        "pivot_refine_workspace_size": ([P, I32, I32, I32], SZ),
        "pivot_decode": ([P, I32, I32, I32, P, P, P, SZ, P], I32),
        "pivot_decode_workspace_size": ([P, I32, I32, I32], SZ),
        "pivot_get_device_error": ([P], I32),
        "pivot_set_wait_limit_ns": ([ctypes.c_uint64], I32),
        "pivot_set_score_buffer_cap": ([SZ], I32),
        "pivot_selftest_wait_timeout": ([P], I32),
        "pivot_status_string": ([I32], ctypes.c_char_p),
        "pivot_version": ([], I32),
        "pivot_profile_enable": ([I32], I32),
        "pivot_profile_read": ([I32, P, P, P], I32),
        "pivot_launch_count": ([], ctypes.c_int64),
        "pivot_decode_noalloc": ([P, I32, I32, I32, P, P, P], I32),
        "pivot_last_error_detail": ([], ctypes.c_char_p),
        "pivot_reuse_backfill": ([I32, I32, I32, P, P, I32, I32, P, P], I32),
        "pivot_window_union": ([P, I32, I32, I32, P, I32, P, P], I32),
        "pivot_index_varlen": ([P, I32, I32, I32, I32, P, P, SZ, P], I32),
        "pivot_index_varlen_workspace_size": ([P, I32, I32, I32, I32], SZ),
        "pivot_index_window_outside": ([P, I32, I32, I32, I32, I32, P, P, SZ, P], I32),
        "pivot_index_window_outside_workspace_size": ([P, I32, I32, I32, I32, I32], SZ),
        "pivot_workspace_size": ([I32, I32, I32, I32, I32, I32, I32, I32, I32], SZ),
        "pivot_set_fused_selection": ([I32, ctypes.c_float], I32),
        "pivot_refine_adaptive": ([P, I32, P, P, I32, I32, ctypes.c_float, P, P, P, P, SZ, P],
                                  I32),
        "pivot_refine_adaptive_workspace_size": ([P, I32, I32, I32], SZ),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


# ---------------------------------------------------------------------------
# C ABI mirrors (same names, same arguments)
# ---------------------------------------------------------------------------

def pivot_dense_index(seq, topk, idx, score, ws, ws_bytes, stream):
    return load().pivot_dense_index(ctypes.byref(seq), topk, idx, score, ws, ws_bytes, stream)


def pivot_dense_index_workspace_size(seq, topk):
    return load().pivot_dense_index_workspace_size(ctypes.byref(seq), topk)


def pivot_proxy_reduce(seq, g, pq, pq_scale, pw, stream):
    return load().pivot_proxy_reduce(ctypes.byref(seq), g, pq, pq_scale, pw, stream)


def pivot_proxy_scan(seq, g, pq, pq_scale, pw, C, topk, cand, cand_score, ws, ws_bytes, stream):
    return load().pivot_proxy_scan(ctypes.byref(seq), g, pq, pq_scale, pw, C, topk, cand,
                                   cand_score, ws, ws_bytes, stream)


def pivot_proxy_scan_workspace_size(seq, g, C):
    return load().pivot_proxy_scan_workspace_size(ctypes.byref(seq), g, C)


def pivot_reuse(t_begin, t_end, g, cand, C, topk, idx, stream):
    return load().pivot_reuse(t_begin, t_end, g, cand, C, topk, idx, stream)


def pivot_reuse_backfill(t_begin, t_end, g, cand, cand_score, C, topk, idx, stream):
    return load().pivot_reuse_backfill(t_begin, t_end, g, cand, cand_score, C, topk, idx, stream)


def pivot_window_union(idx, rows, topk, t_begin, positions, window, out, stream):
    return load().pivot_window_union(idx, rows, topk, t_begin, positions, window, out, stream)


def pivot_refine(seq, g, cand, C, topk, idx, score, ws, ws_bytes, stream):
    return load().pivot_refine(ctypes.byref(seq), g, cand, C, topk, idx, score, ws, ws_bytes,
                               stream)


def pivot_refine_workspace_size(seq, g, C, topk):
    return load().pivot_refine_workspace_size(ctypes.byref(seq), g, C, topk)


def pivot_decode(batch, mode, C, topk, idx, cand, ws, ws_bytes, stream):
    return load().pivot_decode(ctypes.byref(batch), mode, C, topk, idx, cand, ws, ws_bytes,
                               stream)


def pivot_decode_workspace_size(batch, mode, C, topk):
    return load().pivot_decode_workspace_size(ctypes.byref(batch), mode, C, topk)


def pivot_workspace_size(mode, dtype, L_or_maxlen, B, H, D, g, C, topk):
    return load().pivot_workspace_size(mode, dtype, L_or_maxlen, B, H, D, g, C, topk)


def pivot_decode_noalloc(batch, mode, C, topk, idx, cand, stream):
    return load().pivot_decode_noalloc(ctypes.byref(batch), mode, C, topk, idx, cand, stream)


def pivot_get_device_error(stream):
    return load().pivot_get_device_error(stream)


def pivot_set_wait_limit_ns(ns):
    return load().pivot_set_wait_limit_ns(ns)


def pivot_set_score_buffer_cap(nbytes):
    return load().pivot_set_score_buffer_cap(nbytes)


def pivot_set_fused_selection(on, margin_sigmas=4.5):
    return load().pivot_set_fused_selection(on, margin_sigmas)


def pivot_selftest_wait_timeout(stream):
    return load().pivot_selftest_wait_timeout(stream)


def pivot_profile_enable(on):
    return load().pivot_profile_enable(on)


def pivot_profile_read(kernel, launches, total_ms, work):
    return load().pivot_profile_read(kernel, launches, total_ms, work)


def pivot_launch_count():
    return load().pivot_launch_count()


def profile_read(kernel):
    """(launches, total_ms, work) of one kernel class since profiling began."""
    n = ctypes.c_int64(0)
    ms = ctypes.c_double(0.0)
    wk = ctypes.c_double(0.0)
    _check(pivot_profile_read(kernel, ctypes.byref(n), ctypes.byref(ms), ctypes.byref(wk)),
           "pivot_profile_read")
    return n.value, ms.value, wk.value


def pivot_status_string(status):
    return load().pivot_status_string(status).decode()


def pivot_version():
    return load().pivot_version()


def pivot_last_error_detail():
    return load().pivot_last_error_detail().decode()


# ---------------------------------------------------------------------------
# torch marshalling helpers
# ---------------------------------------------------------------------------

def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype in (torch.float8_e4m3fn, torch.uint8):
        return E4M3
    raise TypeError(f"unsupported indexer dtype {t.dtype}")


def _p(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "libpivot takes contiguous CUDA tensors"
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, what):
    if status != 0:
        if status == 4:
            what = f"{what} [{pivot_last_error_detail()}]"
        raise PivotError(status, what)


def _workspace(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def make_seq(q, q_scale, w, k, k_scale, t_begin=0, t_end=0, order=ORDER_POSITION) -> PivotSeq:
    """Describe one prefill sequence; the struct keeps the tensors alive."""
    L, H, D = q.shape
    s = PivotSeq(_dtype_code(q), L, H, D, _p(q), _p(q_scale), _p(w), _p(k), _p(k_scale),
                 t_begin, t_end, order)
    s._keep = (q, q_scale, w, k, k_scale)
    return s


def make_varlen(cu_seqlens, q, q_scale, w, k, k_scale, order=ORDER_POSITION) -> PivotVarlen:
    """Describe a ragged batch: cu_seqlens is a host sequence of nseq + 1
    row offsets; the struct keeps it and the tensors alive."""
    cu = (ctypes.c_int32 * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    _, H, D = q.shape
    s = PivotVarlen(_dtype_code(q), len(cu_seqlens) - 1, H, D, ctypes.addressof(cu), _p(q),
                    _p(q_scale), _p(w), _p(k), _p(k_scale), order)
    s._keep = (cu, q, q_scale, w, k, k_scale)
    return s


def pivot_index_varlen(batch, mode, g, C, topk, idx, ws, ws_bytes, stream):
    return load().pivot_index_varlen(ctypes.byref(batch), mode, g, C, topk, idx, ws, ws_bytes,
                                     stream)


def pivot_index_varlen_workspace_size(batch, mode, g, C, topk):
    return load().pivot_index_varlen_workspace_size(ctypes.byref(batch), mode, g, C, topk)


def pivot_index_window_outside(seq, mode, g, C, topk, window, idx, ws, ws_bytes, stream):
    return load().pivot_index_window_outside(ctypes.byref(seq), mode, g, C, topk, window, idx, ws,
                                             ws_bytes, stream)


def pivot_index_window_outside_workspace_size(seq, mode, g, C, topk, window):
    return load().pivot_index_window_outside_workspace_size(ctypes.byref(seq), mode, g, C, topk,
                                                            window)


def index_window_outside(seq: PivotSeq, mode, g, C, topk, window, ws=None, stream=None,
                         device="cuda"):
    idx = torch.empty(_rows(seq), topk + window, dtype=torch.int32, device=device)
    if ws is None:
        ws = _workspace(pivot_index_window_outside_workspace_size(seq, mode, g, C, topk, window),
                        device)
    _check(pivot_index_window_outside(seq, mode, g, C, topk, window, _p(idx), _p(ws), ws.numel(),
                                      _stream(stream)), "pivot_index_window_outside")
    return idx


def index_varlen(batch: PivotVarlen, mode, g, C, topk, ws=None, stream=None, device="cuda"):
    total = batch._keep[0][batch.nseq]
    idx = torch.empty(total, topk, dtype=torch.int32, device=device)
    if ws is None:
        ws = _workspace(pivot_index_varlen_workspace_size(batch, mode, g, C, topk), device)
    _check(pivot_index_varlen(batch, mode, g, C, topk, _p(idx), _p(ws), ws.numel(),
                              _stream(stream)), "pivot_index_varlen")
    return idx


def make_decode(q, q_scale, w, kc, kc_scale, cache_len, order=ORDER_POSITION) -> PivotDecode:
    """Describe one decode batch; the struct keeps the tensors alive."""
    B, Gm, H, D = q.shape
    s = PivotDecode(_dtype_code(q), B, Gm, H, D, kc.shape[1], _p(q), _p(q_scale), _p(w),
                    _p(kc), _p(kc_scale), _p(cache_len), order)
    s._keep = (q, q_scale, w, kc, kc_scale, cache_len)
    return s


def _rows(seq):
    return (seq.t_end or seq.L) - seq.t_begin


def dense_index(seq: PivotSeq, topk, with_score=False, ws=None, stream=None, device="cuda"):
    n = _rows(seq)
    idx = torch.empty(n, topk, dtype=torch.int32, device=device)
    score = torch.empty(n, topk, dtype=torch.float32, device=device) if with_score else None
    if ws is None:
        ws = _workspace(pivot_dense_index_workspace_size(seq, topk), device)
    _check(pivot_dense_index(seq, topk, _p(idx), _p(score), _p(ws), ws.numel(), _stream(stream)),
           "pivot_dense_index")
    return idx, score


def proxy_reduce(seq: PivotSeq, g, stream=None, device="cuda"):
    G = -(-_rows(seq) // g)
    store = {F32: torch.float32, BF16: torch.bfloat16, E4M3: torch.float8_e4m3fn}[seq.dtype]
    pq = torch.empty(G, seq.H, seq.D, dtype=store, device=device)
    pqs = torch.empty(G, dtype=torch.float32, device=device) if seq.dtype == E4M3 else None
    pw = torch.empty(G, seq.H, dtype=torch.float32, device=device)
    _check(pivot_proxy_reduce(seq, g, _p(pq), _p(pqs), _p(pw), _stream(stream)),
           "pivot_proxy_reduce")
    return pq, pqs, pw


def proxy_scan(seq: PivotSeq, g, pq, pqs, pw, C, topk, with_score=False, ws=None, stream=None,
               device="cuda"):
    """Candidates [G, C]: each proxy's top-topk positions, then the rest of
    its top-C, each ascending (rank order throughout if seq.order asks)."""
    G = pq.shape[0]
    cand = torch.empty(G, C, dtype=torch.int32, device=device)
    cs = torch.empty(G, C, dtype=torch.float32, device=device) if with_score else None
    if ws is None:
        ws = _workspace(pivot_proxy_scan_workspace_size(seq, g, C), device)
    _check(pivot_proxy_scan(seq, g, _p(pq), _p(pqs), _p(pw), C, topk, _p(cand), _p(cs), _p(ws),
                            ws.numel(), _stream(stream)), "pivot_proxy_scan")
    return cand, cs


def reuse(t_begin, t_end, g, cand, topk, stream=None, device="cuda"):
    idx = torch.empty(t_end - t_begin, topk, dtype=torch.int32, device=device)
    _check(pivot_reuse(t_begin, t_end, g, _p(cand), cand.shape[1], topk, _p(idx),
                       _stream(stream)), "pivot_reuse")
    return idx


def reuse_backfill(t_begin, t_end, g, cand, cand_score, topk, stream=None, device="cuda"):
    idx = torch.empty(t_end - t_begin, topk, dtype=torch.int32, device=device)
    _check(pivot_reuse_backfill(t_begin, t_end, g, _p(cand), _p(cand_score), cand.shape[1], topk,
                                _p(idx), _stream(stream)), "pivot_reuse_backfill")
    return idx


def window_union(idx, window, t_begin=0, positions=None, stream=None):
    rows, topk = idx.shape
    out = torch.empty(rows, topk + window, dtype=torch.int32, device=idx.device)
    _check(pivot_window_union(_p(idx), rows, topk, t_begin, _p(positions), window, _p(out),
                              _stream(stream)), "pivot_window_union")
    return out


def refine(seq: PivotSeq, g, cand, topk, with_score=False, ws=None, stream=None, device="cuda"):
    n = _rows(seq)
    C = cand.shape[1]
    idx = torch.empty(n, topk, dtype=torch.int32, device=device)
    score = torch.empty(n, topk, dtype=torch.float32, device=device) if with_score else None
    if ws is None:
        ws = _workspace(pivot_refine_workspace_size(seq, g, C, topk), device)
    _check(pivot_refine(seq, g, _p(cand), C, topk, _p(idx), _p(score), _p(ws), ws.numel(),
                        _stream(stream)), "pivot_refine")
    return idx, score


def pivot_refine_adaptive(seq, g, cand, cand_score, C, topk, rho, cand_count, idx, score, ws,
                          ws_bytes, stream):
    return load().pivot_refine_adaptive(ctypes.byref(seq), g, cand, cand_score, C, topk, rho,
                                        cand_count, idx, score, ws, ws_bytes, stream)


def pivot_refine_adaptive_workspace_size(seq, g, C, topk):
    return load().pivot_refine_adaptive_workspace_size(ctypes.byref(seq), g, C, topk)


def refine_adaptive(seq: PivotSeq, g, cand, cand_score, topk, rho, ws=None, stream=None,
                    device="cuda"):
    """Refine over each group's adaptive count of rank-ordered candidates;
    returns (idx, counts)."""
    n = _rows(seq)
    C = cand.shape[1]
    idx = torch.empty(n, topk, dtype=torch.int32, device=device)
    counts = torch.empty(cand.shape[0], dtype=torch.int32, device=device)
    if ws is None:
        ws = _workspace(pivot_refine_adaptive_workspace_size(seq, g, C, topk), device)
    _check(pivot_refine_adaptive(seq, g, _p(cand), _p(cand_score), C, topk, rho, _p(counts),
                                 _p(idx), None, _p(ws), ws.numel(), _stream(stream)),
           "pivot_refine_adaptive")
    return idx, counts


def decode(batch: PivotDecode, mode, C, topk, want_cand=False, ws=None, stream=None,
           device="cuda"):
    idx = torch.empty(batch.B, batch.Gm, topk, dtype=torch.int32, device=device)
    cand = (torch.empty(batch.B, C, dtype=torch.int32, device=device)
            if (want_cand and mode != DENSE) else None)
    if ws is None:
        ws = _workspace(pivot_decode_workspace_size(batch, mode, C, topk), device)
    _check(pivot_decode(batch, mode, C, topk, _p(idx), _p(cand), _p(ws), ws.numel(),
                        _stream(stream)), "pivot_decode")
    return idx, cand


def device_error(stream=None) -> int:
    return pivot_get_device_error(_stream(stream))


# ---------------------------------------------------------------------------
# cross-layer reuse of index rows
# ---------------------------------------------------------------------------

def layer_anchors(nlayers: int, period: int):
    """Which layer's index rows each of `nlayers` layers uses when every
    `period`-th layer runs the indexer and the layers after it reuse its rows
    (in the style of IndexCache, which the PIVOT blog post names as stacking
    with PIVOT; the pages give none of its method, so the schedule is a plain
    fixed period): anchors[l] = l - l % period."""
    if nlayers < 1 or period < 1:
        raise ValueError("nlayers and period must be >= 1")
    return [layer - layer % period for layer in range(nlayers)]


def index_layers(layer_seqs, mode, g, C, topk, period, stream=None, device="cuda"):
    """Index rows for every layer of a model's consecutive layers: the anchor
    layers (layer_anchors) run the indexer -- dense (mode DENSE) or PIVOT
    with Reuse or Refine -- through the library; every other layer is handed
    its anchor's rows (the same tensor: nothing is recomputed or copied).
    Returns one [rows, topk] int32 tensor per layer."""
    anchors = layer_anchors(len(layer_seqs), period)
    rows = {}
    for layer, seq in enumerate(layer_seqs):
        if anchors[layer] != layer:
            continue
        if mode == DENSE:
            rows[layer], _ = dense_index(seq, topk, stream=stream, device=device)
        else:
            pq, pqs, pw = proxy_reduce(seq, g, stream=stream, device=device)
            cand, _ = proxy_scan(seq, g, pq, pqs, pw, C, topk, stream=stream, device=device)
            t0 = seq.t_begin
            t1 = seq.t_end or seq.L
            rows[layer] = (reuse(t0, t1, g, cand, topk, stream=stream, device=device)
                           if mode == REUSE else
                           refine(seq, g, cand, topk, stream=stream, device=device)[0])
    return [rows[a] for a in anchors]
