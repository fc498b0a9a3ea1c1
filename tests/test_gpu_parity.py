"""Parity of the CUDA path with the CPU oracle, through the C ABI.

Tolerances: the set of chosen experts exact except near-ties (k-th and
(k+1)-th key within 1e-5, which may pick either expert but must stay a valid
top-k); slot order valid (keys descending within 1e-5); routing weights to
1e-5 relative per expert (fp32 against float64); layer output
max|gpu - oracle| / max|oracle| <= 1e-2 for BF16 weights (fp32 accumulate,
BF16 intermediate and output roundings) and <= 3e-2 for FP8.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import moe as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


def _check(rep: gu.Report, fmt: str = "bf16", **kw):
    gu.check(rep, fmt, **kw)


# ------------------------------------------------------------------ tiny layer
@pytest.fixture(scope="module")
def tiny(smoe):
    layer = gu.make_layer(synth.TINY, 300, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=300)
    yield layer, h
    smoe.moe_destroy(h)
    gu.release(layer)


@pytest.mark.parametrize("T", [1, 2, 3, 17, 64, 129, 300])
def test_tiny_bf16(smoe, tiny, T):
    layer, h = tiny
    x = layer.x[:T].contiguous()
    y, ids, w = gu.run(smoe, h, layer, x)
    _check(gu.compare(layer, y, ids, w, x=x))


def test_tiny_forced_routing_all_tokens(smoe, tiny):
    """The oracle's ids fed in: every token's output compares, near-ties too."""
    layer, h = tiny
    r = gu.oracle_route(layer)
    forced = torch.from_numpy(r.ids.astype(np.int32)).cuda()
    y, ids, w = gu.run(smoe, h, layer, forced=forced)
    assert np.array_equal(gu.to_np(ids), r.ids)
    np.testing.assert_allclose(gu.to_np(w), r.weights, rtol=1e-5)
    yo = gu.oracle_outputs(layer, r.ids, r.weights, np.arange(layer.x.shape[0]))
    err = np.max(np.abs(gu.to_np(y) - yo)) / np.max(np.abs(yo))
    assert err <= gu.TOL["bf16"]


def test_tiny_weights_sum_and_bias_only_selects(smoe, tiny):
    layer, h = tiny
    _, ids, w = gu.run(smoe, h, layer)
    np.testing.assert_allclose(gu.to_np(w).sum(axis=1), 2.827, rtol=1e-5)
    assert np.all(gu.to_np(w) > 0)
    ids = gu.to_np(ids)
    assert all(len(set(r)) == len(r) for r in ids.tolist())


def test_identical_experts_closed_form(smoe):
    """All routed experts equal to one SwiGLU E and a zero shared expert:
    y = 2.827 * E(x) whatever the routing."""
    layer = gu.make_layer(synth.TINY, 96, "bf16", identical=True, shared_zero=True)
    h = gu.create_handle(smoe, layer, max_tokens=96)
    try:
        y, _, _ = gu.run(smoe, h, layer)
    finally:
        smoe.moe_destroy(h)
    m = {n: gu.to_np(v).astype(np.float64) for n, v in synth.expert_slice(layer.ew, 0).items()}
    from oracle import moe as orc
    ex = orc.swiglu_expert(gu.to_np(layer.x).astype(np.float64), m["gate"], m["up"], m["down"])
    err = np.max(np.abs(gu.to_np(y) - 2.827 * ex)) / np.max(np.abs(2.827 * ex))
    assert err <= gu.TOL["bf16"]


def test_two_shared_experts(smoe):
    """n_shared_experts = 2: the shared MLP has intermediate 2 * f."""
    shape = synth.LayerShape(hidden_size=256, moe_intermediate_size=128, n_routed_experts=16,
                             num_experts_per_tok=4, n_shared_experts=2)
    layer = gu.make_layer(shape, 70, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=70)
    try:
        y, ids, w = gu.run(smoe, h, layer)
    finally:
        smoe.moe_destroy(h)
    _check(gu.compare(layer, y, ids, w))


def test_no_shared_expert(smoe):
    shape = synth.LayerShape(hidden_size=256, moe_intermediate_size=128, n_routed_experts=16,
                             num_experts_per_tok=4, n_shared_experts=0)
    layer = gu.make_layer(shape, 50, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=50)
    try:
        y, ids, w = gu.run(smoe, h, layer)
    finally:
        smoe.moe_destroy(h)
    _check(gu.compare(layer, y, ids, w))


# ------------------------------------------------------------------ edge cases
def test_edge_cases(smoe, tiny):
    layer, h = tiny
    x = layer.x[:8].contiguous()
    y = torch.full_like(x, 7.0)
    smoe.moe_forward(h, x, y, T=0, flags=smoe.MOE_FLAG_SYNC_CHECK)  # no-op
    assert torch.all(y == 7.0)
    with pytest.raises(smoe.MoeError) as e:
        big = torch.zeros((301, 256), dtype=torch.bfloat16, device="cuda")
        smoe.moe_forward(h, big, torch.empty_like(big))
    assert e.value.status == smoe.MOE_ERR_INVALID_ARG
    with pytest.raises(smoe.MoeError) as e:
        smoe.moe_forward(h, x, x)
    assert e.value.status == smoe.MOE_ERR_INVALID_ARG
    # a forced id out of range: reported through the status word, the forward
    # falls back to selecting, and the handle stays usable
    bad = torch.zeros((8, 4), dtype=torch.int32, device="cuda")
    bad[3] = torch.tensor([0, 1, 2, 99])
    with pytest.raises(smoe.MoeError) as e:
        smoe.moe_forward(h, x, torch.empty_like(x), forced_topk_ids=bad,
                         flags=smoe.MOE_FLAG_SYNC_CHECK)
    assert e.value.status == smoe.MOE_ERR_DEVICE
    assert smoe.moe_get_device_status(h) == 0
    y2, ids, w = gu.run(smoe, h, layer, x)
    _check(gu.compare(layer, y2, ids, w, x=x))


PAIR_LAYER = synth.LayerShape(hidden_size=256, moe_intermediate_size=256, n_routed_experts=16,
                              num_experts_per_tok=4, n_shared_experts=1)


@pytest.mark.parametrize("fmt,shape,T", [
    ("bf16", synth.TINY, 64),    # one-SM BF16 GEMMs (64-row tiles)
    ("bf16", PAIR_LAYER, 300),   # CTA-pair BF16 GEMMs (256-row tiles)
    ("fp8", synth.TINY, 64),     # promoted FP8 GEMMs
])
def test_wait_timeout_winds_down_and_handle_recovers(smoe, fmt, shape, T):
    """The failure path of a GEMM pipeline wait, without a fault: with the
    test stall, the gate/up GEMM's MMA issuer waits on a barrier nothing
    signals, with a 200 us limit. The forward must return MOE_ERR_TIMEOUT
    (the status word read and cleared by the sync check), and the next plain
    forward on the same handle must match the oracle: every CTA let its loads
    land, freed its tensor memory and returned."""
    layer = gu.make_layer(shape, T, fmt)
    h = gu.create_handle(smoe, layer, max_tokens=T)
    try:
        y = torch.empty_like(layer.x)
        with pytest.raises(smoe.MoeError) as e:
            smoe.moe_forward(h, layer.x, y, wait_limit_ns=200_000,
                             flags=smoe.MOE_FLAG_SYNC_CHECK | smoe.MOE_FLAG_TEST_STALL)
        assert e.value.status == smoe.MOE_ERR_TIMEOUT, e.value
        assert smoe.moe_get_device_status(h) == 0  # cleared by the sync check
        for _ in range(2):  # the handle works again, with and without a graph
            r = gu.run(smoe, h, layer)
            gu.check(gu.compare(layer, r.y, r.ids, r.w), fmt)
        y2 = torch.empty_like(layer.x)
        smoe.moe_forward(h, layer.x, y2)
        torch.cuda.synchronize()
        assert torch.equal(y2, r.y)
        assert smoe.moe_get_device_status(h) == 0
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)


def test_forward_rejects_unknown_option_flags(smoe, tiny):
    layer, h = tiny
    x = layer.x[:4].contiguous()
    with pytest.raises(smoe.MoeError) as e:
        smoe.moe_forward(h, x, torch.empty_like(x), flags=0x80)
    assert e.value.status == smoe.MOE_ERR_INVALID_ARG


def test_forward_before_load_is_rejected(smoe):
    cfg = smoe.moe_config_init_k2(hidden_size=256, moe_intermediate_size=128, n_routed_experts=16,
                                  num_experts_per_tok=4, max_tokens=4)
    h = smoe.moe_create(cfg, 0)
    try:
        x = torch.zeros((4, 256), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(smoe.MoeError) as e:
            smoe.moe_forward(h, x, torch.empty_like(x))
        assert e.value.status == smoe.MOE_ERR_STATE
    finally:
        smoe.moe_destroy(h)


def test_host_entry_point_matches_device(smoe, tiny):
    layer, h = tiny
    y_dev, _, _ = gu.run(smoe, h, layer)
    xh = layer.x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    smoe.moe_forward_host(h, xh, yh)
    assert torch.equal(yh, y_dev.cpu())


def test_host_pipeline_matches_device(smoe, tiny):
    """Pipelined host calls (two staging buffers used in turn, uploads and
    downloads on their own streams): each call's result equals moe_forward's
    on the same input, for calls 3 and 4 that reuse calls 1 and 2's staging
    buffers, and for repeated calls on one pair of host buffers."""
    layer, h = tiny
    T = layer.x.shape[0]
    xs = [layer.x, layer.x.flip(0).contiguous(), (layer.x * 0.5).contiguous(),
          layer.x.roll(7, 0).contiguous()]
    want = [gu.run(smoe, h, layer, x)[0].cpu() for x in xs]
    xh = [x.cpu().pin_memory() for x in xs]
    yh = [torch.empty_like(x).pin_memory() for x in xh]
    for i in range(4):
        smoe.moe_forward_host_async(h, xh[i], yh[i])
    smoe.moe_host_wait(h)
    for i in range(4):
        assert torch.equal(yh[i], want[i]), i
    # the same host buffers every call (each download overwrites the last)
    yone = torch.empty_like(xh[0]).pin_memory()
    for i in range(3):
        smoe.moe_forward_host_async(h, xh[1], yone, T=T)
    smoe.moe_host_wait(h)
    assert torch.equal(yone, want[1])


def test_repeated_forwards_replay_a_graph(smoe, tiny):
    """From the second forward with the same (T, x, y) and no options the
    library replays a captured CUDA graph: each result follows the current
    contents of x in the same buffers, equal to a direct forward (one with
    options, which never uses a graph), and the launch count still counts
    the graph's kernels."""
    layer, h = tiny
    scales = (1.0, 0.5, 2.0, -1.0, 0.25)
    want = [gu.run(smoe, h, layer, (layer.x[:64] * c).contiguous())[0].clone() for c in scales]
    x = torch.empty_like(layer.x[:64])
    y = torch.empty_like(x)
    n0 = smoe.moe_launch_count(h)
    for i, c in enumerate(scales):
        x.copy_(layer.x[:64] * c)
        smoe.moe_forward(h, x, y)
        torch.cuda.synchronize()
        assert torch.equal(y, want[i]), i
    assert smoe.moe_launch_count(h) - n0 == len(scales) * 7
    assert smoe.moe_get_device_status(h) == 0


def test_profile_phases(smoe, tiny):
    layer, h = tiny
    smoe.moe_profile_enable(h, 3)
    n0 = smoe.moe_launch_count(h)
    for _ in range(3):
        gu.run(smoe, h, layer)
    ph = smoe.moe_profile_read(h, 3)
    smoe.moe_profile_enable(h, 0)
    assert len(ph) == 3 and all(len(p) == smoe.MOE_NUM_PHASES for p in ph)
    assert all(t >= 0 for p in ph for t in p)
    assert smoe.moe_launch_count(h) - n0 == 3 * 7


# ------------------------------------------------------------------ K2 shapes
@pytest.fixture(scope="module")
def k2(smoe):
    layer = gu.make_layer(synth.K2, 8192, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=8192)
    # one expert-major oracle pass for the tokens every test below compares
    gu.cache_of(layer).prepare(np.union1d(gu.sample_tokens(8192), np.arange(64)),
                               with_ties_below=8192)
    yield layer, h
    smoe.moe_destroy(h)
    gu.release(layer)


def test_k2_decode_T64(smoe, k2):
    """Decode: every one of the 64 tokens compared, and the dispatch's row
    order checked against the routing."""
    layer, h = k2
    x = layer.x[:64].contiguous()
    r = gu.run(smoe, h, layer, x, permutation=True)
    _check(gu.compare(layer, r.y, r.ids, r.w, x=x), min_compared=64)
    print(gu.check_permutation(gu.to_np(r.ids), gu.to_np(r.offsets), gu.to_np(r.pair_rows)))


def test_k2_all_tokens_on_eight_experts(smoe, k2):
    """Maximal imbalance: every token forced onto experts 0..7 (376 experts
    empty, 2048 rows each for the 8, cut into many row tiles): ids as forced,
    weights from the oracle's scores for those ids, outputs of 512 tokens
    (the first and last among them) against the oracle with the same ids and
    weights, and the row order."""
    layer, h = k2
    T, k = 2048, 8
    x = layer.x[:T].contiguous()
    ids = np.tile(np.arange(k, dtype=np.int32), (T, 1))
    forced = torch.from_numpy(ids).cuda()
    r = gu.run(smoe, h, layer, x, forced=forced, permutation=True)
    assert np.array_equal(gu.to_np(r.ids), ids)
    c = gu.cache_of(layer)
    w = orc.routing_weights(c.r.scores[:T], ids.astype(np.int64))
    np.testing.assert_allclose(gu.to_np(r.w), w, rtol=1e-5)
    toks = gu.sample_tokens(T)
    assert len(toks) == 512
    yo = gu.oracle_outputs(layer, ids.astype(np.int64), w, toks, x)
    err = np.max(np.abs(gu.to_np(r.y).astype(np.float64)[toks] - yo)) / np.max(np.abs(yo))
    print(f"eight experts, T={T}: outputs of {len(toks)} tokens, max rel err {err:.2e}")
    assert err <= gu.TOL["bf16"], err
    print(gu.check_permutation(ids, gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    assert smoe.moe_get_device_status(h) == 0


def test_k2_prefill_T8192(smoe, k2):
    """Prefill: routing of all 8192 tokens, outputs of 512 sampled tokens and
    of every near-tie token (under the experts the GPU chose), and the row
    order of all 65,536 (token, slot) pairs."""
    layer, h = k2
    r = gu.run(smoe, h, layer, permutation=True)
    rep = gu.compare(layer, r.y, r.ids, r.w)
    _check(rep)
    ids = gu.to_np(r.ids)
    print(gu.check_permutation(ids, gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    counts = np.bincount(ids.ravel(), minlength=384)
    assert counts.sum() == 8192 * 8 and counts.min() > 0  # ~170 tokens per expert


def test_k2_output_independent_of_batch_kernels(smoe, k2):
    """A token's output must not depend on which GEMM kernels its batch size
    selects: with the same forced experts, the first 512 tokens give the same
    bits at T = 512 (one-SM kernels, 32-row tiles) and at T = 2048 (CTA-pair
    kernels, 128-row tiles). Both sizes use the tensor-core router, whose
    per-token logits do not depend on T, and every GEMM kernel computes
    SwiGLU with the same arithmetic."""
    layer, h = k2
    ids = torch.from_numpy(gu.cache_of(layer).r.ids[:2048].astype(np.int32)).cuda()
    y512 = gu.run(smoe, h, layer, layer.x[:512].contiguous(), forced=ids[:512].contiguous()).y
    y2048 = gu.run(smoe, h, layer, layer.x[:2048].contiguous(), forced=ids).y
    same = (y512 == y2048[:512]).all(dim=1)
    assert bool(same.all()), f"{int((~same).sum())} of 512 tokens differ"


# ------------------------------------------------------------ router logits
@pytest.mark.parametrize("T", [4, 64, 512, 8192])
def test_k2_router_logit_accuracy(smoe, k2, T):
    """Logits from the CUDA-core path (small T) and the tensor-core path
    (T >= 512, fp32 router weight split exactly into three BF16 parts)
    against float64: the error must stay far below the 1e-5 near-tie band
    of the keys (dkey = sigmoid' * dlogit <= dlogit / 4)."""
    layer, h = k2
    x = layer.x[:T].contiguous()
    lg = torch.empty((T, 384), dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    smoe.moe_forward(h, x, y, router_logits_out=lg, flags=smoe.MOE_FLAG_SYNC_CHECK)
    ref = gu.to_np(x).astype(np.float64) @ gu.to_np(layer.Wg).astype(np.float64).T
    err = np.abs(gu.to_np(lg).astype(np.float64) - ref)
    scale = np.abs(gu.to_np(x).astype(np.float64)) @ np.abs(gu.to_np(layer.Wg).astype(np.float64)).T
    print(f"T={T}: max |dlogit| {err.max():.3e}, mean {err.mean():.3e}, "
          f"p99.99 {np.quantile(err, 0.9999):.3e}, max rel to sum|x w| {(err / scale).max():.3e}, "
          f"max |logit| {np.abs(ref).max():.2f}")
    assert err.max() < 2e-5  # key error <= 5e-6, half the near-tie band
