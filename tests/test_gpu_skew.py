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
        y, ids, w = gu.run(smoe, h, layer)
        counts = np.bincount(gu.to_np(ids).ravel(), minlength=384)
        hottest = int(np.argmax(counts))
        rng = np.random.default_rng(4)
        toks = rng.choice(4096, 5, replace=False)
        on_hot = np.nonzero((gu.to_np(ids) == hottest).any(axis=1))[0]
        toks = np.union1d(toks, on_hot[:2])
        rep = gu.compare(layer, y, ids, w, tokens=toks)
    finally:
        smoe.moe_destroy(h)
    assert counts.sum() == 4096 * 8
    assert counts.max() > 800, counts.max()
    assert np.all(counts[scale.numpy() == 0] == 0)
    assert (counts == 0).sum() >= 16
    assert rep.id_mismatch_outside_ties == 0 and rep.invalid_tie_choices == 0, rep
    assert rep.weight_max_rel < 1e-5, rep
    assert rep.y_rel_err <= gu.TOL["bf16"], rep
