"""The proxy and Reuse kernels on the CPU, against the oracle.

csrc/proxy_reuse.cu is compiled by g++ for the host with the CUDA features
it uses emulated (tests/emu; launches run block by block on host threads)
and driven through ctypes (tests/emu/reuse_glue.cpp calls the library's own
launchers).  Checked bit for bit against the oracle: the f32 proxy (mean of
q and w in member order, PIVOT in 10 minutes "How It Works"), including the
packed groups of a ragged batch; Reuse (PIVOT abstract) for prefill, ragged
batches and decode; the window union (indexer tutorial Fig. 3).  The bf16 /
e4m3 stores of the proxy are not emulated (their conversions would abort).
"""
import ctypes
import shutil

import numpy as np
import pytest

import oracle
from emu_build import CSRC, EMU, compile_, prepare, rewrite, rewrite_launches

pytestmark = pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")


@pytest.fixture(scope="module")
def emu(tmp_path_factory):
    d = tmp_path_factory.mktemp("reuse_emu")
    prepare(d, extra=True)
    src = rewrite((CSRC / "proxy_reuse.cu").read_text(),
                  [("extern __shared__ float qbar_s[];", "float* qbar_s = (float*)emu_smem();")])
    (d / "proxy_reuse_emu.cpp").write_text(rewrite_launches(src))
    so = compile_(d, [d / "proxy_reuse_emu.cpp", EMU / "reuse_glue.cpp"], d / "libreuse_emu.so",
                  shared=True)
    lib = ctypes.CDLL(str(so))
    lib.emu_error_word.restype = ctypes.c_uint32
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _cand_rows(rng, G, C, k, ends, L_of):
    """Candidate rows as the proxy scan lays them out: the proxy's top-k
    positions ascending, then the rest of its top-C ascending, -1 padded
    when the prefix [0, e_j] is shorter than C."""
    cand = np.full((G, C), -1, dtype=np.int32)
    for j in range(G):
        n = min(C, ends[j] + 1)
        pick = rng.choice(ends[j] + 1, n, replace=False)
        kk = min(k, n)
        cand[j, :kk] = np.sort(pick[:kk])
        cand[j, kk:n] = np.sort(pick[kk:])
    return cand


@pytest.mark.parametrize("L,g,C,k", [(300, 4, 64, 16), (257, 8, 40, 40), (33, 1, 16, 5)])
def test_reuse_matches_oracle(emu, L, g, C, k):
    rng = np.random.default_rng(L + g)
    G = -(-L // g)
    ends = [min(L, (j + 1) * g) - 1 for j in range(G)]
    cand = _cand_rows(rng, G, C, k, ends, L)
    idx = np.full((L, k), -7, dtype=np.int32)
    assert emu.emu_reuse(0, L, g, _p(cand), C, k, _p(idx), 0, 0) == 0
    assert (idx == oracle.reuse(L, g, cand, k)).all()
    assert emu.emu_error_word() == 0


def test_reuse_ragged_batch_matches_each_sequence(emu):
    rng = np.random.default_rng(5)
    lens = [9, 0, 1, 40, 17, 0, 8]
    g, C, k = 4, 24, 6
    tok = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ng = [-(-n // g) for n in lens]
    grp = np.concatenate([[0], np.cumsum(ng)]).astype(np.int32)
    cands = [_cand_rows(rng, ng[i], C, k, [min(n, (j + 1) * g) - 1 for j in range(ng[i])], n)
             for i, n in enumerate(lens)]
    cand = np.concatenate([c for c in cands if len(c)]).astype(np.int32)
    T = int(tok[-1])
    idx = np.full((T, k), -7, dtype=np.int32)
    assert emu.emu_reuse_varlen(_p(tok), _p(grp), len(lens), T, g, _p(cand), C, k, _p(idx)) == 0
    for i, n in enumerate(lens):
        if n:
            assert (idx[tok[i]:tok[i + 1]] == oracle.reuse(n, g, cands[i], k)).all()
    assert emu.emu_error_word() == 0


def test_decode_reuse_rows(emu):
    """Member m of sequence b keeps the proxy's top-k entries <= cache_len - Gm + m;
    a cache length outside [Gm, maxlen] raises the data error and yields no row."""
    rng = np.random.default_rng(9)
    B, Gm, maxlen, C, k = 5, 3, 64, 20, 8
    cache_len = np.array([3, 64, 17, 2, 40], dtype=np.int32)
    cand = _cand_rows(rng, B, C, k, [max(int(n) - 1, 0) for n in cache_len], None)
    idx = np.full((B * Gm, k), -7, dtype=np.int32)
    assert emu.emu_decode_reuse(B, Gm, maxlen, _p(cache_len), _p(cand), C, k, _p(idx)) == 0
    assert emu.emu_error_word() == 2                       # sequence 3: 2 < Gm
    for b in range(B):
        for m in range(Gm):
            row = idx[b * Gm + m]
            if cache_len[b] < Gm:
                assert (row == -1).all()
                continue
            lim = int(cache_len[b]) - Gm + m
            want = [c for c in cand[b, :k] if 0 <= c <= lim]
            assert list(row[:len(want)]) == want and (row[len(want):] == -1).all()


@pytest.mark.parametrize("window", [1, 3, 50])
def test_window_union_matches_oracle(emu, window):
    rng = np.random.default_rng(window)
    rows, k = 120, 10
    idx = np.full((rows, k), -1, dtype=np.int32)
    for t in range(rows):
        n = min(k, t + 1)
        idx[t, :n] = np.sort(rng.choice(t + 1, n, replace=False))
    out = np.full((rows, k + window), -7, dtype=np.int32)
    assert emu.emu_window_union(_p(idx), rows, k, 0, None, window, _p(out), 0) == 0
    assert (out == oracle.window_union_rows(idx, 0, window)).all()
    # in place: rows at stride k + window, the first k entries holding the index row
    buf = np.full((rows, k + window), -7, dtype=np.int32)
    buf[:, :k] = idx
    assert emu.emu_window_union(_p(buf), rows, k, 0, None, window, _p(buf), k + window) == 0
    assert (buf == out).all()


@pytest.mark.parametrize("ragged", [False, True])
def test_f32_proxy_matches_oracle(emu, ragged):
    rng = np.random.default_rng(3)
    H, D, g = 4, 32, 3
    lens = [10, 0, 1, 7] if ragged else [11]
    parts = [(rng.standard_normal((n, H, D)).astype(np.float32),
              rng.random((n, H)).astype(np.float32)) for n in lens]
    q = np.concatenate([p[0] for p in parts]).astype(np.float32)
    w = np.concatenate([p[1] for p in parts]).astype(np.float32)
    tok = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ng = [-(-n // g) for n in lens]
    grp = np.concatenate([[0], np.cumsum(ng)]).astype(np.int32)
    G = int(grp[-1])
    pq = np.zeros((G, H, D), dtype=np.float32)
    pw = np.zeros((G, H), dtype=np.float32)
    rc = emu.emu_proxy_reduce_f32(_p(q), _p(w), int(tok[-1]), H, D, g, G, _p(pq), _p(pw),
                                  _p(tok) if ragged else None, _p(grp) if ragged else None,
                                  len(lens))
    assert rc == 0 and emu.emu_error_word() == 0
    for i, (qi, wi) in enumerate(parts):
        if not len(qi):
            continue
        opq, _, opw = oracle.proxy_reduce(oracle.F32, qi, None, wi, g)
        assert np.array_equal(pq[grp[i]:grp[i + 1]], np.asarray(opq, dtype=np.float32))
        assert np.array_equal(pw[grp[i]:grp[i + 1]], np.asarray(opw, dtype=np.float32))


def test_table_copy_by_launch_parameters(emu):
    host = np.arange(960, dtype=np.int32) * 7 - 3
    dst = np.zeros(960, dtype=np.int32)
    assert emu.emu_write_ints(_p(dst), _p(host), 960) == 0
    assert (dst == host).all()
    assert emu.emu_write_ints(_p(dst), _p(host), 961) != 0        # above the limit: refused
