"""Group-limited routing (n_group > 1) on the GPU against the oracle.

K2 sets n_group = topk_group = 1 ("Kimi K2 Base" raw config; "Behind
Kimi-K2's Config" §2.4 explains that grouping balances load inside a device
and why K2 drops it). The library also runs the grouped router of the
DeepSeek-V3-shaped layers it descends from, with this library's reading of
the group rule: contiguous groups of E / n_group experts, a group scores the
fp32 sum of its two largest selection keys, the topk_group best groups are
kept (ties to the lower group), the top-k runs over their experts only.

Same acceptance rule as the other parity tests; a token is also a near-tie
when its kept and next group scores are within 2e-5, and may then keep the
other group (the choice must stay valid).
"""
import numpy as np
import pytest

import synth
from oracle import moe as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

TINY_GROUPED = synth.LayerShape(hidden_size=256, moe_intermediate_size=128, n_routed_experts=16,
                                num_experts_per_tok=4, n_shared_experts=1, n_group=4,
                                topk_group=2)
# DeepSeek-V3-shaped router: 256 experts in 8 groups, 4 groups kept, top-8,
# hidden 7168 (small experts keep the test cheap; the router is the subject)
DSV3_ROUTER = synth.LayerShape(hidden_size=7168, moe_intermediate_size=256, n_routed_experts=256,
                               num_experts_per_tok=8, n_shared_experts=1, n_group=8,
                               topk_group=4)


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


def _grouping_matters(layer, T):
    """Tokens whose grouped choice differs from the plain top-k: the filter
    must be exercised, not a no-op."""
    c = gu.cache_of(layer)
    s = layer.shape
    plain = orc.route(c.x[:T], gu.f64(layer.Wg), gu.f64(layer.b), s.num_experts_per_tok)
    return sum(set(a) != set(b) for a, b in zip(plain.ids, c.r.ids[:T]))


@pytest.mark.parametrize("T", [1, 5, 64, 300])
def test_tiny_grouped(smoe, T):
    layer = gu.make_layer(TINY_GROUPED, 300, "bf16", bias_std=0.05)
    h = gu.create_handle(smoe, layer, max_tokens=300)
    try:
        x = layer.x[:T].contiguous()
        r = gu.run(smoe, h, layer, x)
        gu.check(gu.compare(layer, r.y, r.ids, r.w, x=x))
        ids = gu.to_np(r.ids)
        assert all(len(set((ids[t] // 4).tolist())) <= 2 for t in range(T))
        if T >= 64:
            assert _grouping_matters(layer, T) > T // 10
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)


@pytest.fixture(scope="module")
def dsv3(smoe):
    layer = gu.make_layer(DSV3_ROUTER, 2048, "bf16", bias_std=0.05)
    h = gu.create_handle(smoe, layer, max_tokens=2048)
    yield layer, h
    smoe.moe_destroy(h)
    gu.release(layer)


@pytest.mark.parametrize("T", [4, 64, 2048])  # GEMV, split-K and tensor-core routers
def test_dsv3_shaped_grouped_router(smoe, dsv3, T):
    layer, h = dsv3
    x = layer.x[:T].contiguous()
    r = gu.run(smoe, h, layer, x, permutation=True)
    rep = gu.compare(layer, r.y, r.ids, r.w, x=x)
    gu.check(rep)
    ids = gu.to_np(r.ids)
    assert all(len(set((ids[t] // 32).tolist())) <= 4 for t in range(T))
    print(gu.check_permutation(ids, gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    if T >= 64:
        n = _grouping_matters(layer, T)
        print(f"T={T}: {n} tokens choose differently from the plain top-k")
        assert n > T // 20
