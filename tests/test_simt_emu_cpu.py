"""The CUDA-core scoring kernels (csrc/simt.cu) on the CPU.

They score shapes outside the tensor-core tiling (H not dividing 256, key
rows not 128 or 256 bytes) and small Refine member blocks.  The source is
compiled by g++ with the CUDA features emulated (tests/emu) and driven
through its launchers.  On integer inputs every score is exact in fp32, so
each written entry must equal the indexer score of the indexer tutorial
(Fig. 1-2, in its multi-head form with head weights and ReLU) bit for bit,
and no entry past a row's causal limit may be written: prefill rows, proxy
rows (limit = the group's last member), MTP decode rows over ragged cache
lengths, and Refine rows over candidate keys.
"""
import ctypes
import shutil

import numpy as np
import pytest

from emu_build import CSRC, EMU, compile_, prepare, rewrite, rewrite_launches

F32, BF16 = 0, 1
PREFILL_DENSE, PREFILL_PROXY, DECODE_DENSE, DECODE_PROXY = 0, 1, 2, 3
SENTINEL = np.float32(-12345.0)

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    d = tmp_path_factory.mktemp("simt_emu")
    prepare(d, extra=True)
    src = (CSRC / "simt.cu").read_text()
    assert src.count("extern __shared__ float sm[];") == 2
    src = src.replace("extern __shared__ float sm[];", "float* sm = (float*)emu_smem();")
    (d / "simt_emu.cpp").write_text(rewrite_launches(src))
    so = compile_(d, [d / "simt_emu.cpp", EMU / "simt_glue.cpp"], d / "libsimt_emu.so",
                  shared=True)
    lib = ctypes.CDLL(str(so))
    lib.emu_error_word.restype = ctypes.c_uint32
    lib.emu_scan_simt.argtypes = [ctypes.c_int] * 5 + [ctypes.c_void_p] * 5 + \
        [ctypes.c_int] * 4 + [ctypes.c_void_p] + [ctypes.c_int] * 4 + [ctypes.c_void_p, ctypes.c_longlong]
    lib.emu_refine_simt.argtypes = [ctypes.c_int] * 4 + [ctypes.c_void_p] * 4 + \
        [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2 + [ctypes.c_int] * 4 + [ctypes.c_void_p]
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _ints(rng, shape, lo, hi):
    return rng.integers(lo, hi + 1, size=shape).astype(np.float32)


def _score(q, w, k):
    """I(r, s) = sum_h w[r,h] * max(0, q[r,h] . k[s]) for all r, s (fp64; exact here)."""
    dots = np.einsum("rhd,sd->rhs", q.astype(np.float64), k.astype(np.float64))
    return np.einsum("rh,rhs->rs", w.astype(np.float64), np.maximum(dots, 0.0))


def _stored(x, dtype):
    """The codes the kernel reads: fp32 as is, bf16 as the top half (values exact)."""
    if dtype == F32:
        return np.ascontiguousarray(x, dtype=np.float32)
    return np.ascontiguousarray((x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))


@pytest.mark.parametrize("dtype,H,D,P", [(F32, 3, 20, 8), (BF16, 5, 24, 8), (F32, 1, 7, 3)])
def test_prefill_and_proxy_rows_exact(emu, dtype, H, D, P):
    rng = np.random.default_rng(H * 100 + D)
    L, g = 300, 3
    q, k, w = _ints(rng, (L, H, D), -3, 3), _ints(rng, (L, D), -3, 3), _ints(rng, (L, H), 1, 4)
    qc, kc = _stored(q, dtype), _stored(k, dtype)
    stride = 320
    full = _score(q, w, k)
    # dense rows, in two launches (rows [0, 137) and [137, L))
    S = np.full((L, stride), SENTINEL, dtype=np.float32)
    for r0, r1 in ((0, 137), (137, L)):
        assert emu.emu_scan_simt(PREFILL_DENSE, dtype, H, D, P, _p(qc), None, _p(w), _p(kc), None,
                                 L, 1, 1, 0, None, r0, r1 - r0, 0, r1 - 1,
                                 _p(S[r0:]), stride) == 0
    for t in range(L):
        assert np.array_equal(S[t, :t + 1], full[t, :t + 1].astype(np.float32)), t
        assert (S[t, t + 1:] == SENTINEL).all(), t
    # proxy rows: row j = group j's query, limit = min(L, (j+1) g) - 1
    G = -(-L // g)
    pq, pw = q[:G], w[:G]
    Sp = np.full((G, stride), SENTINEL, dtype=np.float32)
    assert emu.emu_scan_simt(PREFILL_PROXY, dtype, H, D, P, _p(_stored(pq, dtype)), None, _p(pw),
                             _p(kc), None, L, g, 1, 0, None, 0, G, 0, L - 1, _p(Sp), stride) == 0
    fp = _score(pq, pw, k)
    for j in range(G):
        e = min(L, (j + 1) * g) - 1
        assert np.array_equal(Sp[j, :e + 1], fp[j, :e + 1].astype(np.float32)), j
        assert (Sp[j, e + 1:] == SENTINEL).all(), j
    assert emu.emu_error_word() == 0


def test_decode_rows_exact_and_bad_lengths(emu):
    """Member m of sequence b scores keys [0, cache_len[b] - Gm + m] of its own
    cache; a length outside [Gm, maxlen] writes nothing and raises no fault
    here (the selection reports it)."""
    rng = np.random.default_rng(4)
    B, Gm, H, D, maxlen = 4, 2, 3, 12, 200
    cache_len = np.array([2, 200, 77, 1], dtype=np.int32)           # the last is invalid
    q, w = _ints(rng, (B * Gm, H, D), -3, 3), _ints(rng, (B * Gm, H), 1, 4)
    kc = _ints(rng, (B, maxlen, D), -3, 3)
    S = np.full((B * Gm, maxlen), SENTINEL, dtype=np.float32)
    assert emu.emu_scan_simt(DECODE_DENSE, F32, H, D, Gm, _p(q), None, _p(w), _p(kc.reshape(-1, D)),
                             None, 0, 1, Gm, maxlen, _p(cache_len), 0, B * Gm, 0, maxlen - 1,
                             _p(S), maxlen) == 0
    for b in range(B):
        for m in range(Gm):
            r = b * Gm + m
            n = int(cache_len[b])
            if n < Gm:
                assert (S[r] == SENTINEL).all()
                continue
            lim = n - Gm + m
            want = _score(q[r:r + 1], w[r:r + 1], kc[b])[0, :lim + 1].astype(np.float32)
            assert np.array_equal(S[r, :lim + 1], want) and (S[r, lim + 1:] == SENTINEL).all()


@pytest.mark.parametrize("g,C", [(3, 40), (5, 130), (1, 17)])
def test_refine_rows_exact(emu, g, C):
    """Member t re-scores its group's candidate keys: entry c holds the score
    against key cand[j][c] when 0 <= cand[j][c] <= t; nothing else is written."""
    rng = np.random.default_rng(g * 7 + C)
    L, H, D = 150, 3, 20
    q, k, w = _ints(rng, (L, H, D), -3, 3), _ints(rng, (L, D), -3, 3), _ints(rng, (L, H), 1, 4)
    G = -(-L // g)
    cand = np.full((G, C), -1, dtype=np.int32)
    for j in range(G):
        e = min(L, (j + 1) * g) - 1
        n = min(C, e + 1)
        cand[j, :n] = np.sort(rng.choice(e + 1, n, replace=False))
    S = np.full((L, C), SENTINEL, dtype=np.float32)
    assert emu.emu_refine_simt(PREFILL_DENSE, F32, H, D, _p(q), None, _p(w), _p(k), L, g, 1, 0,
                               None, _p(cand), 0, C, 0, L, _p(S)) == 0
    full = _score(q, w, k)
    for t in range(L):
        row = cand[t // g]
        for c in range(C):
            pos = int(row[c])
            if 0 <= pos <= t:
                assert S[t, c] == np.float32(full[t, pos]), (t, c)
            else:
                assert S[t, c] == SENTINEL, (t, c)
