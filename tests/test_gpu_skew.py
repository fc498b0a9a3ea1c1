"""Skewed routing at K2 shapes: T = 4096 tokens, correction bias ~N(0, 0.05),
router rows scaled (tests/golden/skew_router_scale.txt, written by
make_skew_router.py from the oracle's routing) so that expert popularity is
heavy-tailed: the hottest expert takes over 800 tokens (many row tiles), and
the 16 zero rows leave their experts empty (no work units at all). Parity on
sampled tokens plus the routing of every token, as for the other workloads."""
import os

import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "skew_router_scale.txt")


def skew_scale() -> torch.Tensor:
    vals = [float(l) for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    assert len(vals) == 384
    return torch.tensor(vals, dtype=torch.float32)


def test_skewed_routing_parity_and_imbalance():
    import sparse_moe_sigmoid_b200 as smoe
    scale = skew_scale()
    layer = gu.make_layer(synth.K2, 4096, "bf16", router_row_scale=scale, bias_std=0.05)
    h = gu.create_handle(smoe, layer, max_tokens=4096)
    try:
        r = gu.run(smoe, h, layer, permutation=True)
        ids = gu.to_np(r.ids)
        counts = np.bincount(ids.ravel(), minlength=384)
        hottest = int(np.argmax(counts))
        # 512 sampled tokens, plus the first and last rows of the hottest
        # expert (its first and last row tiles)
        on_hot = np.nonzero((ids == hottest).any(axis=1))[0]
        toks = np.union1d(gu.sample_tokens(4096), np.concatenate([on_hot[:4], on_hot[-4:]]))
        rep = gu.compare(layer, r.y, r.ids, r.w, tokens=toks)
        perm = gu.check_permutation(ids, gu.to_np(r.offsets), gu.to_np(r.pair_rows))
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)
    print(perm)
    assert counts.sum() == 4096 * 8
    assert counts.max() > 800, counts.max()
    assert np.all(counts[scale.numpy() == 0] == 0)
    assert (counts == 0).sum() >= 16
    gu.check(rep, "bf16")
