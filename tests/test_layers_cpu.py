"""Cross-layer reuse of index rows, host side: the layer schedule and the
correlated synthetic layers (no GPU)."""
import numpy as np
import pytest
import torch

import oracle
from top_token_selection_b200 import inputs as gen
from top_token_selection_b200 import pivot as pv


def test_layer_anchors():
    assert pv.layer_anchors(5, 1) == [0, 1, 2, 3, 4]
    assert pv.layer_anchors(5, 2) == [0, 0, 2, 2, 4]
    assert pv.layer_anchors(4, 9) == [0, 0, 0, 0]
    with pytest.raises(ValueError):
        pv.layer_anchors(0, 2)
    with pytest.raises(ValueError):
        pv.layer_anchors(3, 0)


def test_layers_keep_the_generator_and_correlate_by_rho():
    same = gen.make_layers(3, 256, 4, 32, gen.F32, rho=1.0, seed=1)
    for layer in same[1:]:
        assert torch.equal(layer.q, same[0].q) and torch.equal(layer.k, same[0].k)
        assert torch.equal(layer.w, same[0].w)
    for rho in (0.0, 0.8):
        lay = gen.make_layers(2, 4096, 4, 32, gen.F32, rho=rho, seed=2)
        a, b = lay[0].k.flatten().numpy(), lay[1].k.flatten().numpy()
        assert abs(np.corrcoef(a, b)[0, 1] - rho) < 0.05
        # marginals stay the generator's (unit-variance keys up to the heavy 2%)
        assert abs(b.std() / a.std() - 1.0) < 0.1


def test_reuse_recall_grows_with_correlation():
    """By the oracle: the rows a layer reuses from the layer before cover
    more of its own dense top-k when the layers correlate more (and all of
    it when they are identical)."""
    L, H, D, kk = 300, 4, 32, 32
    rows = np.arange(100, L, 20)
    recall = {}
    for rho in (1.0, 0.95, 0.3):
        lay = gen.make_layers(2, L, H, D, gen.F32, rho=rho, seed=3)
        idx = []
        for p in lay:
            q, qs, w, k, ks = p.codes()
            idx.append(oracle.dense_index(gen.F32, q, qs, w, k, ks, kk, rows=rows)[0])
        recall[rho] = np.mean([len(set(a) & set(b)) / kk for a, b in zip(idx[0], idx[1])])
    assert recall[1.0] == 1.0
    assert recall[0.95] > recall[0.3]
