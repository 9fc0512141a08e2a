"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad arguments before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

from top_token_selection_b200 import build as pbuild
from top_token_selection_b200 import pivot as pv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pivot.h")


@pytest.fixture(scope="module")
def lib():
    pbuild.build()
    return pv.load()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pivot_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert header_functions() == sorted(pv.ABI_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", pv.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (pivot_\w+)", out))
    missing = [f for f in header_functions() if f not in exported]
    assert not missing, missing
    for f in header_functions():
        assert hasattr(lib, f)


def test_version_and_status_strings(lib):
    assert pv.pivot_version() == 100
    assert pv.pivot_status_string(0) == "ok"
    assert pv.pivot_status_string(3) == "workspace too small"


FAKE = 0x10000   # never dereferenced: every call below fails validation first


def _seq(**kw):
    base = dict(dtype=pv.F32, L=64, H=4, D=32, q=FAKE, q_scale=None, w=FAKE, k=FAKE,
                k_scale=None, t_begin=0, t_end=0)
    base.update(kw)
    return pv.PivotSeq(**base)


@pytest.mark.parametrize("bad", [
    dict(dtype=7), dict(L=0), dict(H=0), dict(q=None), dict(w=None), dict(k=None),
    dict(q_scale=FAKE),                       # f32 takes no scales
    dict(dtype=pv.E4M3, D=128),               # e4m3 needs both scales
    dict(t_begin=10, t_end=5), dict(t_end=65), dict(q=FAKE + 4),
])
def test_dense_rejects_bad_sequences(lib, bad):
    seq = _seq(**bad)
    st = pv.pivot_dense_index(seq, 8, FAKE, None, FAKE, 1 << 20, None)
    assert st == 1, bad


def test_dense_rejects_bad_topk_and_workspace(lib):
    seq = _seq()
    assert pv.pivot_dense_index(seq, 0, FAKE, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_dense_index(seq, 8, None, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_dense_index(seq, 8, FAKE, None, None, 1 << 20, None) == 1
    assert pv.pivot_dense_index(seq, 8, FAKE, None, FAKE + 16, 1 << 20, None) == 1  # alignment
    assert pv.pivot_dense_index(seq, 8, FAKE, None, FAKE, 64, None) == 3            # too small
    assert pv.pivot_dense_index(seq, 1 << 20, FAKE, None, FAKE, 1 << 20, None) == 2


def test_group_and_candidate_checks(lib):
    seq = _seq(t_begin=3)
    assert pv.pivot_proxy_reduce(seq, 4, FAKE, None, FAKE, None) == 1      # t_begin % g
    seq = _seq()
    assert pv.pivot_proxy_reduce(seq, 0, FAKE, None, FAKE, None) == 1      # g >= 1
    assert pv.pivot_proxy_reduce(seq, 4, FAKE, FAKE, FAKE, None) == 1      # no pq_scale for f32
    assert pv.pivot_proxy_scan(seq, 4, FAKE, None, FAKE, 0, 1, FAKE, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_proxy_scan(seq, 4, FAKE, None, FAKE, 8, 9, FAKE, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_proxy_scan(seq, 4, FAKE, None, FAKE, 8, 0, FAKE, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_reuse(0, 64, 4, FAKE, 8, 16, FAKE, None) == 1           # C < k
    assert pv.pivot_reuse(1, 64, 4, FAKE, 16, 8, FAKE, None) == 1           # t_begin % g
    assert pv.pivot_refine(seq, 4, FAKE, 8, 16, FAKE, None, FAKE, 1 << 20, None) == 1


def test_workspace_sizes(lib):
    seq = _seq(L=1000, H=4, D=32)
    n = pv.pivot_dense_index_workspace_size(seq, 64)
    assert n >= 1000 * 1024 * 4 and n % 256 == 0
    assert pv.pivot_proxy_scan_workspace_size(seq, 4, 256) >= 250 * 1024 * 4
    assert pv.pivot_refine_workspace_size(seq, 4, 256, 64) >= 1000 * 256 * 4
    assert pv.pivot_dense_index_workspace_size(_seq(L=0), 64) == 0
    dec = pv.PivotDecode(pv.E4M3, 4, 2, 64, 128, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert pv.pivot_decode_workspace_size(dec, pv.DENSE, 0, 64) >= 8 * 4096 * 4
    assert pv.pivot_decode_workspace_size(dec, pv.REFINE, 256, 64) > \
        pv.pivot_decode_workspace_size(dec, pv.REUSE, 256, 64)
    assert pv.pivot_decode_workspace_size(dec, pv.REUSE, 32, 64) == 0      # C < k


def test_missing_library_fails_loudly(tmp_path):
    saved = pv._lib
    try:
        pv._lib = None
        with pytest.raises(ImportError):
            pv.load(str(tmp_path / "nope.so"))
    finally:
        pv._lib = saved


def test_next_steps_reject_bad_arguments(lib):
    assert pv.pivot_reuse_backfill(0, 64, 0, FAKE, FAKE, 16, 8, FAKE, None) == 1    # g >= 1
    assert pv.pivot_reuse_backfill(3, 64, 4, FAKE, FAKE, 16, 8, FAKE, None) == 1    # t_begin % g
    assert pv.pivot_reuse_backfill(0, 64, 4, FAKE, None, 16, 8, FAKE, None) == 1    # scores needed
    assert pv.pivot_reuse_backfill(0, 64, 4, FAKE, FAKE, 8, 16, FAKE, None) == 1    # C < k
    assert pv.pivot_reuse_backfill(0, 64, 4, FAKE, FAKE, 1 << 20, 8, FAKE, None) == 2
    assert pv.pivot_window_union(FAKE, 4, 8, 0, None, 0, FAKE, None) == 1          # window >= 1
    assert pv.pivot_window_union(FAKE, 4, 0, 0, None, 3, FAKE, None) == 1          # topk >= 1
    assert pv.pivot_window_union(None, 4, 8, 0, None, 3, FAKE, None) == 1
    assert pv.pivot_window_union(FAKE, 4, 8, -1, None, 3, FAKE, None) == 1         # no positions
    assert pv.pivot_window_union(FAKE, 0, 8, 0, None, 3, FAKE, None) == 0          # nothing to do


def test_ragged_batch_rejects_bad_arguments(lib):
    import ctypes

    def batch(cu):
        arr = (ctypes.c_int32 * len(cu))(*cu)
        b = pv.PivotVarlen(pv.F32, len(cu) - 1, 4, 32, ctypes.addressof(arr), FAKE, None, FAKE,
                           FAKE, None)
        b._keep = (arr,)
        return b
    good = batch([0, 10, 30])
    assert pv.pivot_index_varlen_workspace_size(good, 1, 4, 16, 8) > 0
    assert pv.pivot_index_varlen(batch([0, 10, 5]), 0, 4, 16, 8, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_varlen(batch([1, 10]), 0, 4, 16, 8, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_varlen(good, 3, 4, 16, 8, FAKE, FAKE, 1 << 20, None) == 1    # mode
    assert pv.pivot_index_varlen(good, 1, 4, 8, 16, FAKE, FAKE, 1 << 20, None) == 1    # C < k
    assert pv.pivot_index_varlen(good, 1, 0, 16, 8, FAKE, FAKE, 1 << 20, None) == 1    # g
    assert pv.pivot_index_varlen(good, 1, 4, 16, 8, FAKE, FAKE, 64, None) == 3         # workspace
    assert pv.pivot_index_varlen(good, 1, 4, 16, 8, FAKE, FAKE + 16, 1 << 20, None) == 1
    assert pv.pivot_index_varlen_workspace_size(batch([0, 10, 5]), 0, 4, 16, 8) == 0


def test_window_outside_rejects_bad_arguments(lib):
    seq = _seq()
    assert pv.pivot_index_window_outside(seq, 0, 4, 16, 8, 0, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_window_outside(seq, 3, 4, 16, 8, 4, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_window_outside(seq, 1, 4, 8, 16, 4, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_window_outside(seq, 1, 0, 16, 8, 4, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_window_outside(seq, 0, 4, 16, 8, 4, None, FAKE, 1 << 20, None) == 1
    assert pv.pivot_index_window_outside(seq, 0, 4, 16, 8, 4, FAKE, FAKE, 64, None) == 3
    assert pv.pivot_index_window_outside_workspace_size(seq, 2, 4, 16, 8, 4) > 0
    assert pv.pivot_index_window_outside_workspace_size(seq, 2, 4, 16, 8, 0) == 0


def test_score_buffer_cap_shrinks_workspaces(lib):
    """The score-buffer cap bounds what the workspace functions ask for (the
    calls then work in several launches); 0 restores the default, and caps
    below 4096 bytes are refused."""
    import ctypes
    seq = _seq(L=1000, H=4, D=32)
    cu = [0, 700, 0 + 700, 1900]
    arr = (ctypes.c_int32 * len(cu))(*cu)
    batch = pv.PivotVarlen(pv.E4M3, len(cu) - 1, 64, 128, ctypes.addressof(arr), FAKE, FAKE,
                           FAKE, FAKE, FAKE)
    batch._keep = (arr,)
    full = (pv.pivot_dense_index_workspace_size(seq, 64),
            pv.pivot_index_varlen_workspace_size(batch, 0, 8, 256, 64),
            pv.pivot_index_varlen_workspace_size(batch, 2, 8, 256, 64))
    assert pv.pivot_set_score_buffer_cap(100) == 1
    try:
        assert pv.pivot_set_score_buffer_cap(1 << 16) == 0
        small = (pv.pivot_dense_index_workspace_size(seq, 64),
                 pv.pivot_index_varlen_workspace_size(batch, 0, 8, 256, 64),
                 pv.pivot_index_varlen_workspace_size(batch, 2, 8, 256, 64))
        for a, b in zip(small, full):
            assert 0 < a < b and a % 256 == 0
    finally:
        assert pv.pivot_set_score_buffer_cap(0) == 0
    assert (pv.pivot_dense_index_workspace_size(seq, 64),
            pv.pivot_index_varlen_workspace_size(batch, 0, 8, 256, 64),
            pv.pivot_index_varlen_workspace_size(batch, 2, 8, 256, 64)) == full


def test_ragged_batch_workspace_layout(lib):
    """One-launch ragged batch (tensor-core shape): the workspace holds the
    four segment tables, proxies and candidates of every group, and one
    score buffer at the longest sequence's stride; a shape outside the
    tensor-core tiling sizes for the sequence-by-sequence path instead."""
    import ctypes
    lens = [700, 0, 1200, 1, 9]
    cu = [0]
    for n in lens:
        cu.append(cu[-1] + n)
    arr = (ctypes.c_int32 * len(cu))(*cu)

    def batch(H, D, dtype):
        b = pv.PivotVarlen(dtype, len(lens), H, D, ctypes.addressof(arr), FAKE,
                           FAKE if dtype == pv.E4M3 else None, FAKE, FAKE,
                           FAKE if dtype == pv.E4M3 else None)
        b._keep = (arr,)
        return b
    g, C, k = 8, 256, 64
    T, G, maxL = sum(lens), sum(-(-n // g) for n in lens), max(lens)
    up = lambda x: -(-x // 256) * 256
    tabs = up(4 * (len(lens) + 1) * 4)
    prox = up(G * 64 * 128) + up(G * 4) + up(G * 64 * 4) + up(G * C * 4)
    stride = -(-maxL // 32) * 32
    dense_rows = up(T * (stride * 4 + 4))
    b = batch(64, 128, pv.E4M3)
    assert pv.pivot_index_varlen_workspace_size(b, 0, g, C, k) == tabs + dense_rows
    assert pv.pivot_index_varlen_workspace_size(b, 1, g, C, k) == tabs + prox + up(G * (stride * 4 + 4))
    refine_s = max(G * (stride * 4 + 4), T * C * 4)
    assert pv.pivot_index_varlen_workspace_size(b, 2, g, C, k) == tabs + prox + up(refine_s)
    # H = 2 is not a tensor-core shape: the sequence-by-sequence layout
    seq_path = pv.pivot_index_varlen_workspace_size(batch(2, 64, pv.F32), 0, g, C, k)
    assert 0 < seq_path < T * (stride * 4 + 4)


def test_one_workspace_size_for_a_whole_pass(lib):
    """pivot_workspace_size from sizes alone equals the largest per-call
    workspace of the mode's chain (prefill with B = 0, decode with B >= 1)."""
    for dt, D, scale in ((pv.F32, 32, None), (pv.E4M3, 128, FAKE), (pv.BF16, 128, None)):
        H = 4 if dt == pv.F32 else 64
        seq = _seq(dtype=dt, L=5000, H=H, D=D, q_scale=scale, k_scale=scale)
        dense = pv.pivot_dense_index_workspace_size(seq, 256)
        scan = pv.pivot_proxy_scan_workspace_size(seq, 8, 1024)
        ref = pv.pivot_refine_workspace_size(seq, 8, 1024, 256)
        assert pv.pivot_workspace_size(pv.DENSE, dt, 5000, 0, H, D, 8, 1024, 256) == dense
        assert pv.pivot_workspace_size(pv.REUSE, dt, 5000, 0, H, D, 8, 1024, 256) == scan
        assert pv.pivot_workspace_size(pv.REFINE, dt, 5000, 0, H, D, 8, 1024, 256) == max(scan, ref)
    dec = pv.PivotDecode(pv.E4M3, 4, 2, 64, 128, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        assert pv.pivot_workspace_size(mode, pv.E4M3, 4096, 4, 64, 128, 2, 256, 64) == \
            pv.pivot_decode_workspace_size(dec, mode, 256, 64)
    # arguments the calls refuse give 0
    assert pv.pivot_workspace_size(3, pv.F32, 5000, 0, 4, 32, 8, 1024, 256) == 0
    assert pv.pivot_workspace_size(pv.REUSE, pv.F32, 5000, 0, 4, 32, 8, 100, 256) == 0   # C < k
    assert pv.pivot_workspace_size(pv.DENSE, 9, 5000, 0, 4, 32, 8, 1024, 256) == 0


def test_output_order_field_is_validated(lib):
    """order is PIVOT_ORDER_POSITION (0) or PIVOT_ORDER_RANK (1); anything
    else is an invalid argument for every call that reads it."""
    for order in (2, -1):
        seq = _seq(order=order)
        assert pv.pivot_dense_index(seq, 8, FAKE, None, FAKE, 1 << 20, None) == 1
        assert pv.pivot_proxy_scan(seq, 4, FAKE, None, FAKE, 16, 8, FAKE, None, FAKE, 1 << 20,
                                   None) == 1
        assert pv.pivot_refine(seq, 4, FAKE, 16, 8, FAKE, None, FAKE, 1 << 20, None) == 1
        dec = pv.PivotDecode(pv.E4M3, 4, 2, 64, 128, 4096, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                             order)
        assert pv.pivot_decode(dec, pv.DENSE, 0, 64, FAKE, None, FAKE, 1 << 20, None) == 1
        cu = (ctypes.c_int32 * 2)(0, 64)
        vb = pv.PivotVarlen(pv.F32, 1, 4, 32, ctypes.addressof(cu), FAKE, None, FAKE, FAKE, None,
                            order)
        assert pv.pivot_index_varlen(vb, pv.DENSE, 4, 16, 8, FAKE, FAKE, 1 << 20, None) == 1
    assert pv.pivot_dense_index_workspace_size(_seq(order=pv.ORDER_RANK), 8) > 0


def test_fused_selection_hook(lib):
    """The fused-selection switch takes 0 or 1 and a finite margin; switching
    it off sizes the score buffer path's workspace instead."""
    seq = _seq(dtype=pv.E4M3, L=20000, H=64, D=128, q_scale=FAKE, k_scale=FAKE)
    try:
        assert pv.pivot_set_fused_selection(2, 4.5) == 1
        assert pv.pivot_set_fused_selection(1, float("nan")) == 1
        assert pv.pivot_set_fused_selection(1, 4.5) == 0
        fused = pv.pivot_dense_index_workspace_size(seq, 2048)
        assert pv.pivot_set_fused_selection(0, 4.5) == 0
        plain = pv.pivot_dense_index_workspace_size(seq, 2048)
        assert fused > 0 and plain > 0 and fused != plain
    finally:
        assert pv.pivot_set_fused_selection(0, 4.5) == 0   # the default


def test_adaptive_refine_rejects_bad_arguments(lib):
    seq = _seq()
    ws = pv.pivot_refine_adaptive_workspace_size(seq, 4, 16, 8)
    assert ws > pv.pivot_refine_workspace_size(seq, 4, 16, 8)
    for rho in (-0.1, 1.5, float("nan")):
        assert pv.pivot_refine_adaptive(seq, 4, FAKE, FAKE, 16, 8, rho, None, FAKE, None, FAKE,
                                        1 << 20, None) == 1
    assert pv.pivot_refine_adaptive(seq, 4, FAKE, None, 16, 8, 0.5, None, FAKE, None, FAKE,
                                    1 << 20, None) == 1           # no candidate scores
    assert pv.pivot_refine_adaptive(seq, 4, FAKE, FAKE, 8, 16, 0.5, None, FAKE, None, FAKE,
                                    1 << 20, None) == 1           # C < k
