"""pivot_decode_noalloc: the decode step for callers that cannot allocate.

Some callers cannot hand the library a workspace -- a plugin inside an
inference engine whose memory planner owns the whole device, or a decode
loop that may not allocate in the middle of its per-token step.  For them
the library runs the decode step with a fixed scratch array of its own.
These tests check, through the C ABI, that it returns what the regular
pivot_decode returns with a caller workspace, on calls in a row with
batches of different shapes (the array keeps the previous call's contents,
so a later call's scratch lands on stale data at shifted offsets), and that
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


def _batch(seed, dtype, B=6, Gm=2, len_lo=500, len_hi=6000):
    d = gen.make_decode(B=B, Gm=Gm, H=64, D=128, dtype=dtype, len_lo=len_lo, len_hi=len_hi,
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


def _same_as_decode(batch, mode, C, topk, what):
    want_idx, want_cand = pv.decode(batch, mode, C, topk, want_cand=True)
    got_idx, got_cand = _noalloc(batch, mode, C, topk)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    # same kernels on the same inputs: identical index rows (this is within
    # any tolerance the other parity tests use)
    assert torch.equal(got_idx, want_idx), what
    if mode != pv.DENSE:
        assert torch.equal(got_cand, want_cand), what


@pytest.mark.parametrize("dtype", [gen.E4M3, gen.BF16])
def test_noalloc_decode_matches_decode_with_workspace(dtype):
    # Call 1: a large dense step whose score rows fill the front of the
    # shared array; then calls of another shape (fewer sequences, three MTP
    # tokens, shorter caches, other C and k), whose scratch layout lands on
    # the stale contents at different offsets.
    big = _batch(11, dtype, B=16, Gm=2, len_lo=20000, len_hi=60000)
    _same_as_decode(big, pv.DENSE, 0, 2048, "large dense")
    small = _batch(12, dtype, B=3, Gm=3, len_lo=300, len_hi=2500)
    for mode in (pv.REUSE, pv.REFINE, pv.DENSE):
        _same_as_decode(small, mode, 256, 64, ("small", mode))
    # and back to the configuration sizes (C = 4096, k = 2048)
    for mode in (pv.REFINE, pv.REUSE):
        _same_as_decode(big, mode, 4096, 2048, ("large", mode))


def test_noalloc_rejects_a_batch_beyond_its_scratch():
    # One sequence with an (8M + 4096)-key cache: two dense score rows need
    # just over 64 MiB, more than the array holds, so the call is refused
    # before anything is enqueued.  The buffers are real and the cached
    # length is short, so nothing could read out of bounds even if the size
    # guard were lost.
    maxlen = (1 << 23) + 4096
    dev = "cuda"
    q = torch.zeros((1, 2, 64, 128), dtype=torch.float8_e4m3fn, device=dev)
    qs = torch.ones((1, 2), dtype=torch.float32, device=dev)
    w = torch.ones((1, 2, 64), dtype=torch.float32, device=dev)
    kc = torch.zeros((1, maxlen, 128), dtype=torch.float8_e4m3fn, device=dev)
    kcs = torch.ones((1, maxlen), dtype=torch.float32, device=dev)
    cl = torch.tensor([1000], dtype=torch.int32, device=dev)
    big = pv.make_decode(q, qs, w, kc, kcs, cl)
    assert pv.pivot_decode_workspace_size(big, pv.DENSE, 0, 128) > 64 << 20
    idx = torch.full((1, 2, 128), -7, dtype=torch.int32, device=dev)
    st = pv.pivot_decode_noalloc(big, pv.DENSE, 0, 128, idx.data_ptr(), None, None)
    assert st == 3, pv.pivot_status_string(st)     # PIVOT_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert (idx == -7).all()                        # nothing ran
    # the argument checks are pivot_decode's: a null output is an invalid
    # argument, an oversized k unsupported, for both entry points
    assert pv.pivot_decode_noalloc(big, pv.DENSE, 0, 128, None, None, None) == 1
    assert pv.pivot_decode_noalloc(big, pv.DENSE, 0, 9000, idx.data_ptr(), None, None) == 2
    assert pv.pivot_decode(big, pv.DENSE, 0, 9000, idx.data_ptr(), None, None, 0, None) == 2
    del kc, kcs
    small = _batch(13, gen.E4M3)
    got, _ = _noalloc(small, pv.DENSE, 0, 64)       # still usable afterwards
    torch.cuda.synchronize()
    assert pv.device_error() == 0 and (got >= -1).all()
