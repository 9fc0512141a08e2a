"""The selection kernels on the CPU: csrc/topk.cu compiled for the host with
the CUDA features it uses emulated (tests/emu: one thread per CUDA thread,
block barriers, warp collectives, dynamic shared memory filled with junk),
under AddressSanitizer and UndefinedBehaviorSanitizer.  Every row must equal
a plain sort's top-k by (score desc, position asc), listed by position --
the selection rule of the indexer tutorial (Fig. 1: the top-k positions of
the scores) with the tie and order readings of this library.

The kernel source is used as it is; only its launch syntax and shared-memory
declarations are rewritten for the host, and the few helpers it takes from
common.cuh are copied from there verbatim.
"""
import re
import shutil
import subprocess

import pytest

from emu_build import CSRC, EMU, compile_, prepare, rewrite

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


@pytest.fixture(scope="module")
def select_check(tmp_path_factory):
    d = tmp_path_factory.mktemp("select_emu")
    prepare(d)
    topk = rewrite((CSRC / "topk.cu").read_text(), [
        ("extern __shared__ __align__(16) uint8_t smem[];", "uint8_t* smem = emu_smem();"),
        ("select_kernel<<<p.nrows, SEL_THREADS, lay.total, stream>>>(p);",
         "emu_launch(p.nrows, SEL_THREADS, lay.total, [&] { select_kernel(p); });"),
        ("extern __shared__ __align__(16) uint8_t smem_t[];", "uint8_t* smem_t = emu_smem();"),
        ("row_threshold_kernel<<<grid, THR_WARPS * 32, smem, stream>>>(p, thresh);",
         "emu_launch(grid, THR_WARPS * 32, smem, [&] { row_threshold_kernel(p, thresh); });"),
        ("extern __shared__ __align__(16) uint8_t smem_b[];", "uint8_t* smem_b = emu_smem();"),
        ("sample_bound_kernel<<<(p.nrows + FB_WARPS - 1) / FB_WARPS, FB_WARPS * 32, smem, stream>>>(p);",
         "emu_launch((p.nrows + FB_WARPS - 1) / FB_WARPS, FB_WARPS * 32, smem, "
         "[&] { sample_bound_kernel(p); });"),
        ("extern __shared__ __align__(16) uint8_t smem_f[];", "uint8_t* smem_f = emu_smem();"),
        ("fused_finish_kernel<<<(p.nrows + warps - 1) / warps, warps * 32, smem, stream>>>(p, warps);",
         "emu_launch((p.nrows + warps - 1) / warps, warps * 32, smem, "
         "[&] { fused_finish_kernel(p, warps); });"),
    ])
    (d / "topk_emu.cpp").write_text(topk)
    return compile_(d, [d / "topk_emu.cpp", EMU / "select_check.cpp"], d / "select_check",
                    sanitize=True)


@pytest.fixture(scope="module")
def select_check_debug(tmp_path_factory, select_check):
    """The same harness with PIVOT_DEBUG defined: the kernels' own index
    checks are on."""
    d = select_check.parent
    return compile_(d, [d / "topk_emu.cpp", EMU / "select_check.cpp"], d / "select_check_debug",
                    sanitize=True, defines=("PIVOT_DEBUG",))


def _run(exe, *args):
    res = subprocess.run([str(exe), *map(str, args)], capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, (res.stdout + res.stderr)[-4000:]
    assert res.stdout.strip().endswith("0 bad rows, error word 0")


@pytest.mark.parametrize("L,K,split,dist,rows,bound", [
    (20000, 2048, 0, 0, 3, 1),      # sampled bound, buffer path
    (20000, 2048, 1024, 0, 2, 1),   # a candidate row: the top 1024 listed first
    (9000, 300, 0, 1, 3, 1),        # five distinct values: ties decided by position
    (9000, 64, 0, 2, 3, 0),         # signed zeros, bound sampled inside the select
    (20000, 1, 0, 3, 2, 1),         # k = 1 under a heavy tail
    (20000, 4096, 2048, 1, 3, 1),   # k = 4096 with a split: the trimmed boundary buffer, ties
    # rows to 128K (4096 bitmap words): proxy rows (k = 4096, the top 2048
    # first) in two CTAs' shared memory, with and without ties at the k-th
    (131072, 4096, 2048, 0, 2, 1),
    (131072, 4096, 2048, 4, 2, 1),
    (131072, 2048, 0, 4, 2, 1),
    (20000, 4096, 2048, 5, 3, 1),   # one value everywhere: both split searches see one value
])
def test_prefix_rows_match_a_sort(select_check, L, K, split, dist, rows, bound):
    _run(select_check, "prefix", L, K, split, dist, rows, bound)


@pytest.mark.parametrize("mode", [0, 1, 2, 3])
def test_candidate_rows_match_a_sort(select_check, mode):
    """Refine rows (the block select, candidate rows in place): cand[j] gives the
    positions, the member's limit masks later ones; ties (1), -1 padded rows
    (2), per-key scales multiplied in (3)."""
    _run(select_check, "cand", 4096, 2048, mode, 9, 0, 0)


@pytest.mark.parametrize("C,K,mode,order,layout", [
    (4096, 2048, 1, 1, 0),   # rank order with heavy ties
    (4096, 2048, 3, 1, 0),   # rank order, per-key scales
    (4096, 2048, 0, 0, 1),   # shuffled candidate rows: sorted by position, not merged
    (300, 300, 1, 0, 0),     # C = k, ties
    (40, 9, 2, 0, 0),        # tiny rows, -1 padding
    (8192, 2048, 0, 0, 0),   # C = 8192 > twice k: compacted above the sampled bound
    (8192, 8192, 1, 1, 1),   # k = C = 8192, rank order, shuffled
    (10000, 2048, 1, 0, 0),  # C = 10000: above the in-place capacity, compacted
    (10000, 2048, 3, 1, 1),  # the same in rank order, shuffled, per-key scales
    (1, 1, 0, 0, 0),         # one candidate
])
def test_candidate_rows_orders_and_sizes(select_check, C, K, mode, order, layout):
    _run(select_check, "cand", C, K, mode, 7, order, layout)


@pytest.mark.parametrize("kind,g,K,C", [(0, 8, 64, 0), (1, 8, 16, 96), (2, 8, 16, 96),
                                        (0, 3, 1, 0), (2, 3, 40, 40)])
def test_ragged_batch_rows_match_a_sort(select_check, kind, g, K, C):
    """Rows of a packed ragged batch (sequences of 0 to 300 tokens) mapped
    through the segment tables -- dense rows, proxy rows (top C, the top K
    first) and member candidate rows with per-sequence key scales -- at each
    sequence's edges, where a mapping error would show."""
    _run(select_check, "varlen", kind, g, K, C)


@pytest.mark.parametrize("kind,K", [(0, 64), (1, 300)])
def test_decode_rows_match_a_sort(select_check, kind, K):
    """MTP decode rows over ragged cache lengths: member m of a sequence sees
    [0, cache_len - Gm + m], the proxy [0, cache_len - 1]; a length outside
    [Gm, maxlen] gives a -1 row and raises the data error."""
    _run(select_check, "decode", kind, K)


@pytest.mark.parametrize("L,g,C,K", [(40, 4, 12, 5), (33, 8, 30, 30)])
def test_backfill_rows_match_a_sort(select_check, L, g, C, K):
    """Reuse with backfill (the reading this library takes where the PIVOT
    abstract's Reuse leaves masked slots open): member t takes the top K of
    its group's candidates at or before t by proxy score, lower position
    first on ties (scores drawn from six values, so ties are common)."""
    _run(select_check, "backfill", L, g, C, K)


@pytest.mark.parametrize("L,K,split,dist,rows,r0,order,sigmas,kind,want_fallback", [
    (20000, 2048, 0, 0, 6, 19990, 0, 4.5, 0, "none"),    # long dense rows, normal scores
    (20000, 2048, 0, 0, 5, 3000, 0, 4.5, 0, "none"),     # rows within the capacity keep all
    (20000, 2048, 0, 3, 5, 19000, 1, 4.5, 0, "none"),    # heavy tail, rank order
    (20000, 100, 0, 1, 6, 15000, 0, 4.5, 0, "any"),      # five values: ties at the bound
    (20000, 2048, 0, 0, 4, 19000, 0, -40.0, 0, "all"),   # bound too high: every row falls back
    (20000, 2048, 0, 0, 4, 19000, 1, 400.0, 0, "all"),   # bound too low: every row falls back
    (40000, 4096, 2048, 0, 4, 4990, 0, 4.5, 1, "none"),  # proxy rows: top-k first, then the rest
    (40000, 4096, 2048, 0, 3, 4990, 0, -40.0, 1, "all"), # the same through the fallback
    (40000, 4096, 2048, 2, 3, 4990, 1, -40.0, 1, "any"), # signed zeros and small integers
    (262144, 2048, 0, 0, 2, 262142, 0, 4.5, 0, "none"),  # rows spanning four bitmap windows
    (40000, 8192, 0, 0, 2, 39990, 0, 4.5, 0, "none"),    # k = 8192: capacity 16384
    (40000, 8192, 0, 1, 2, 39990, 1, -40.0, 0, "all"),   # the same through the fallback
])
def test_fused_selection_matches_a_sort(select_check, L, K, split, dist, rows, r0, order, sigmas,
                                        kind, want_fallback):
    """The selection fused into the scan: sample bound, warp select of the
    survivors and, for rows that miss it, the keep-everything fallback --
    every row equals a plain sort."""
    res = subprocess.run([str(select_check), "fused", *map(str, (L, K, split, dist, rows, r0, order,
                                                                  sigmas, kind))],
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, (res.stdout + res.stderr)[-4000:]
    m = re.search(r"fallback rows (\d+) of (\d+)", res.stdout)
    n_fb, n = int(m.group(1)), int(m.group(2))
    if want_fallback == "none":
        assert n_fb == 0
    elif want_fallback == "all":
        assert n_fb == n


@pytest.mark.parametrize("args", [("prefix", 20000, 2048, 0, 0, 3, 1), ("cand", 4096, 2048, 1, 5, 0, 0),
                                  ("fused", 20000, 2048, 0, 0, 4, 19000, 0, 4.5, 0),
                                  ("fused", 40000, 4096, 2048, 0, 3, 4990, 0, -40.0, 1)])
def test_debug_build_raises_nothing_on_valid_rows(select_check_debug, args):
    """PIVOT_DEBUG build: valid rows pass every check (error word 0) and
    select exactly as the normal build does."""
    _run(select_check_debug, *args)


def test_debug_build_flags_a_planted_bitmap_overrun(select_check_debug):
    """A launch whose bitmap is sized for 64 positions while the row reaches
    20000: the debug build skips every out-of-range bitmap access (no
    sanitizer report) and raises the bounds bit (4) in the error word."""
    res = subprocess.run([str(select_check_debug), "planted", "20000", "2048", "64"],
                         capture_output=True, text=True, timeout=600)
    assert "ERROR: AddressSanitizer" not in res.stderr, res.stderr[-3000:]
    assert res.stdout.strip().endswith("error word 4"), res.stdout + res.stderr[-2000:]
