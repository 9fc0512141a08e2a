"""Cross-layer reuse of index rows on the GPU: anchor layers run the
indexer through the library, the layers after them are handed the anchor's
rows (the same tensor)."""
import pytest
import torch

from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv

from parity import seq_of, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pv.load()


@pytest.mark.parametrize("mode", [pv.DENSE, pv.REUSE, pv.REFINE])
def test_index_layers_reuses_anchor_rows(mode):
    lay = gen.make_layers(4, 3000, 64, 128, gen.E4M3, rho=0.9, seed=5)
    seqs = [seq_of(to_device(p)) for p in lay]
    g, C, kk = 8, 512, 128
    rows = pv.index_layers(seqs, mode, g, C, kk, period=2)
    torch.cuda.synchronize()
    assert pv.device_error() == 0
    assert rows[1] is rows[0] and rows[3] is rows[2]
    for a in (0, 2):   # an anchor's rows are its own indexer call's
        if mode == pv.DENSE:
            want, _ = pv.dense_index(seqs[a], kk)
        else:
            pq, pqs, pw = pv.proxy_reduce(seqs[a], g)
            cand, _ = pv.proxy_scan(seqs[a], g, pq, pqs, pw, C, kk)
            want = (pv.reuse(0, 3000, g, cand, kk) if mode == pv.REUSE
                    else pv.refine(seqs[a], g, cand, kk)[0])
        assert torch.equal(rows[a], want)
