"""pivot_decode_noalloc: the decode step for callers that cannot allocate.

Some callers cannot hand the library a workspace -- a plugin inside an
inference engine whose memory planner owns the whole device, or a decode
loop that may not allocate in the middle of its per-token step.  For them
the library runs the decode step with a fixed scratch array of its own.
These tests check, through the C ABI, that it returns what the regular
pivot_decode returns with a caller workspace, on two calls in a row with
different batches (the array keeps the previous call's contents), and that
a batch too large for the array is refused before anything runs.

This file is named to be collected last.
"""
import ctypes

import pytest
import torch

from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


def _batch(seed, dtype):
    d = gen.make_decode(B=6, Gm=2, H=64, D=128, dtype=dtype, len_lo=500, len_hi=6000,
                        seed=seed)
    c = "cuda"
    return pv.make_decode(d.q.to(c), None if d.q_scale is None else d.q_scale.to(c),
                          d.w.to(c), d.kc.to(c), None if d.kc_scale is None else d.kc_scale.to(c),
                          d.cache_len.to(c))


def _noalloc(batch, mode, C, topk):
    idx = torch.full((batch.B, batch.Gm, topk), -7, dtype=torch.int32, device="cuda")
    cand = (torch.full((batch.B, C), -7, dtype=torch.int32, device="cuda")
            if mode != pv.DENSE else None)
    st = pv.pivot_decode_noalloc(batch, mode, C, topk, idx.data_ptr(),
                                 None if cand is None else cand.data_ptr(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, pv.pivot_status_string(st)
    return idx, cand


@pytest.mark.parametrize("dtype", [gen.E4M3, gen.BF16])
def test_noalloc_decode_matches_decode_with_workspace(dtype):
    C, topk = 512, 128
    for call, seed in enumerate((11, 12)):          # two calls in a row, different batches
        batch = _batch(seed, dtype)
        for mode in (pv.DENSE, pv.REUSE, pv.REFINE):
            want_idx, want_cand = pv.decode(batch, mode, C, topk, want_cand=True)
            got_idx, got_cand = _noalloc(batch, mode, C, topk)
            torch.cuda.synchronize()
            assert pv.device_error() == 0
            # same kernels on the same inputs: identical index rows (this is
            # within any tolerance the other parity tests use)
            assert torch.equal(got_idx, want_idx), (call, mode)
            if mode != pv.DENSE:
                assert torch.equal(got_cand, want_cand), (call, mode)


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    # 64 sequences of 1M cached keys need 512 MiB of dense scores: refused
    # before anything is enqueued, so the (never dereferenced) pointers below
    # are not touched.
    fake = 1 << 20
    big = pv.PivotDecode(pv.E4M3, 64, 2, 64, 128, 1 << 20, fake, fake, fake, fake, fake, fake)
    assert pv.pivot_decode_workspace_size(big, pv.DENSE, 0, 128) > 64 << 20
    st = pv.pivot_decode_noalloc(big, pv.DENSE, 0, 128, fake, None, None)
    assert st == 3, pv.pivot_status_string(st)     # PIVOT_ERR_WORKSPACE
    small = _batch(13, gen.E4M3)
    idx, _ = _noalloc(small, pv.DENSE, 0, 64)       # still usable afterwards
    torch.cuda.synchronize()
    assert pv.device_error() == 0 and (idx >= -1).all()
