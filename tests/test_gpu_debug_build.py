"""The bounds-checking build (libpivot_debug.so, PIVOT_DEBUG): every kernel
checks its own index invariants and reports a failed check through the
device error word instead of trapping.  On valid inputs it must raise
nothing and return exactly what the normal build returns: dense, proxy scan,
Refine and decode on FP8 inputs, through the fused selection and its forced
rescan.
"""
import ctypes
import os

import pytest
import torch

from top_token_selection_b200 import build as libbuild
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dbg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()
    path = libbuild.build(debug=True)
    lib = ctypes.CDLL(path)
    P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.pivot_dense_index.argtypes = [P, I32, P, P, P, SZ, P]
    lib.pivot_dense_index_workspace_size.argtypes = [P, I32]
    lib.pivot_dense_index_workspace_size.restype = SZ
    lib.pivot_proxy_scan.argtypes = [P, I32, P, P, P, I32, I32, P, P, P, SZ, P]
    lib.pivot_proxy_scan_workspace_size.argtypes = [P, I32, I32]
    lib.pivot_proxy_scan_workspace_size.restype = SZ
    lib.pivot_refine.argtypes = [P, I32, P, I32, I32, P, P, P, SZ, P]
    lib.pivot_refine_workspace_size.argtypes = [P, I32, I32, I32]
    lib.pivot_refine_workspace_size.restype = SZ
    lib.pivot_decode.argtypes = [P, I32, I32, I32, P, P, P, SZ, P]
    lib.pivot_decode_workspace_size.argtypes = [P, I32, I32, I32]
    lib.pivot_decode_workspace_size.restype = SZ
    lib.pivot_get_device_error.argtypes = [P]
    lib.pivot_set_fused_selection.argtypes = [I32, ctypes.c_float]
    assert os.path.basename(path) == "libpivot_debug.so"
    yield lib
    lib.pivot_set_fused_selection(0, 4.5)


def _ws(n):
    return torch.empty(max(int(n), 256), dtype=torch.uint8, device="cuda")


@pytest.mark.parametrize("sig", [4.5, -60.0])
def test_debug_build_matches_and_raises_nothing(dbg, sig):
    L, g, C, kk = 6000, 8, 1024, 256
    p = gen.make_prefill(L, 64, 128, gen.E4M3, kind="dsa", seed=4)
    dev = to_device(p)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for order in (pv.ORDER_POSITION, pv.ORDER_RANK):
        seq = pv.make_seq(dev["q"], dev["q_scale"], dev["w"], dev["k"], dev["k_scale"],
                          order=order)
        want_d, _ = pv.dense_index(seq, kk)
        pq, pqs, pw = pv.proxy_reduce(seq, g)
        want_c, _ = pv.proxy_scan(seq, g, pq, pqs, pw, C, kk)
        want_r, _ = pv.refine(seq, g, want_c, kk)
        assert dbg.pivot_set_fused_selection(1, sig) == 0
        got_d = torch.empty_like(want_d)
        ws = _ws(dbg.pivot_dense_index_workspace_size(ctypes.byref(seq), kk))
        assert dbg.pivot_dense_index(ctypes.byref(seq), kk, got_d.data_ptr(), None, ws.data_ptr(),
                                     ws.numel(), st) == 0
        got_c = torch.empty_like(want_c)
        ws = _ws(dbg.pivot_proxy_scan_workspace_size(ctypes.byref(seq), g, C))
        assert dbg.pivot_proxy_scan(ctypes.byref(seq), g, pq.data_ptr(), pqs.data_ptr(),
                                    pw.data_ptr(), C, kk, got_c.data_ptr(), None, ws.data_ptr(),
                                    ws.numel(), st) == 0
        got_r = torch.empty_like(want_r)
        ws = _ws(dbg.pivot_refine_workspace_size(ctypes.byref(seq), g, C, kk))
        assert dbg.pivot_refine(ctypes.byref(seq), g, got_c.data_ptr(), C, kk, got_r.data_ptr(),
                                None, ws.data_ptr(), ws.numel(), st) == 0
        torch.cuda.synchronize()
        assert dbg.pivot_get_device_error(st) == 0          # no check failed
        assert pv.device_error() == 0
        assert torch.equal(got_d, want_d) and torch.equal(got_c, want_c)
        assert torch.equal(got_r, want_r)
    dbg.pivot_set_fused_selection(0, 4.5)


def test_debug_build_decode(dbg):
    d = gen.make_decode(B=4, Gm=2, H=64, D=128, dtype=gen.E4M3, len_lo=2000, len_hi=12000, seed=8)
    c = "cuda"
    batch = pv.make_decode(d.q.to(c), d.q_scale.to(c), d.w.to(c), d.kc.to(c), d.kc_scale.to(c),
                           d.cache_len.to(c))
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
        want, _ = pv.decode(batch, mode, 1024, 256)
        got = torch.empty_like(want)
        ws = _ws(dbg.pivot_decode_workspace_size(ctypes.byref(batch), mode, 1024, 256))
        assert dbg.pivot_decode(ctypes.byref(batch), mode, 1024, 256, got.data_ptr(), None,
                                ws.data_ptr(), ws.numel(), st) == 0
        torch.cuda.synchronize()
        assert dbg.pivot_get_device_error(st) == 0
        assert torch.equal(got, want), mode
