"""The single-launch layer for small batches against the oracle.

With single_launch_max_tokens set, batches of up to 128 tokens whose row
tiles are 16 rows run the whole layer as one cooperative kernel (router, top-k, scan, placement, both GEMMs in one
pipeline, combine, with bounded grid barriers between the phases). These
tests hold it to the same acceptance rule as the phase kernels (routing of
every token, outputs of every token, near-ties under the GPU's choice), check
that it is one launch, that it agrees with the phase kernels
(MOE_FLAG_PHASE_KERNELS), that its profiler phases come from device
timestamps, and that a stalled pipeline returns MOE_ERR_TIMEOUT with the
handle usable afterwards.
"""
import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


def _one_launch(smoe, h, x):
    n0 = smoe.moe_launch_count(h)
    y = torch.empty_like(x)
    smoe.moe_forward(h, x, y, flags=smoe.MOE_FLAG_SYNC_CHECK)
    return smoe.moe_launch_count(h) - n0


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
@pytest.mark.parametrize("T", [1, 5, 16])
def test_tiny_single_launch(smoe, fmt, T):
    layer = gu.make_layer(synth.TINY, 16, fmt)
    h = gu.create_handle(smoe, layer, max_tokens=16, single_launch_max_tokens=128)
    try:
        x = layer.x[:T].contiguous()
        assert _one_launch(smoe, h, x) == 1
        r = gu.run(smoe, h, layer, x, permutation=True)
        gu.check(gu.compare(layer, r.y, r.ids, r.w, x=x), fmt)
        print(gu.check_permutation(gu.to_np(r.ids), gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)


@pytest.fixture(scope="module", params=["bf16", "fp8"])
def k2small(smoe, request):
    fmt = request.param
    layer = gu.make_layer(synth.K2, 128, fmt)
    h = gu.create_handle(smoe, layer, max_tokens=128, single_launch_max_tokens=128)
    gu.cache_of(layer).prepare(np.arange(128), with_ties_below=128)
    yield layer, h, fmt
    smoe.moe_destroy(h)
    gu.release(layer)


@pytest.mark.parametrize("T", [1, 16, 64, 128])
def test_k2_single_launch(smoe, k2small, T):
    layer, h, fmt = k2small
    x = layer.x[:T].contiguous()
    assert _one_launch(smoe, h, x) == 1
    r = gu.run(smoe, h, layer, x, permutation=True)
    gu.check(gu.compare(layer, r.y, r.ids, r.w, x=x), fmt, min_compared=T)
    print(gu.check_permutation(gu.to_np(r.ids), gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    # against the phase kernels: the same experts outside near-ties, outputs
    # within the tolerance of each other
    p = gu.run(smoe, h, layer, x, flags=smoe.MOE_FLAG_PHASE_KERNELS)
    tie = gu.cache_of(layer).r.margin[:T] < gu.NEAR_TIE
    same = np.array([set(a) == set(b) for a, b in zip(gu.to_np(r.ids), gu.to_np(p.ids))])
    assert np.all(same | tie)
    ok = same
    a, b = gu.to_np(r.y)[ok], gu.to_np(p.y)[ok]
    assert np.max(np.abs(a - b)) / np.max(np.abs(b)) <= gu.TOL[fmt]
    assert smoe.moe_get_device_status(h) == 0


def test_k2_single_launch_graph_and_profile(smoe, k2small):
    """Repeated plain forwards replay the one-launch graph; the profiler's
    phases come from the kernel's own timestamps and cover the forward."""
    layer, h, fmt = k2small
    x = layer.x[:64].contiguous()
    want = gu.run(smoe, h, layer, x).y
    y = torch.empty_like(x)
    n0 = smoe.moe_launch_count(h)
    for _ in range(3):
        smoe.moe_forward(h, x, y)
    torch.cuda.synchronize()
    assert torch.equal(y, want)
    assert smoe.moe_launch_count(h) - n0 == 3
    smoe.moe_profile_enable(h, 2)
    for _ in range(2):
        smoe.moe_forward(h, x, y)
    ph = smoe.moe_profile_read(h, 2)
    smoe.moe_profile_enable(h, 0)
    for p in ph:
        assert all(t >= 0 for t in p) and p[4] > 0 and p[5] == 0  # both GEMMs in phase 4
        assert sum(p) < 50.0
    print("phases (ms):", [round(t, 4) for t in ph[-1]])


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_single_launch_timeout_winds_down(smoe, fmt):
    """The stalled MMA issuer of the single launch: MOE_ERR_TIMEOUT, the
    status word cleared, and the next forwards on the handle match the
    oracle (every CTA left the grid barriers, drained its loads and freed
    its tensor memory)."""
    layer = gu.make_layer(synth.TINY, 8, fmt)
    h = gu.create_handle(smoe, layer, max_tokens=8, single_launch_max_tokens=128)
    try:
        y = torch.empty_like(layer.x)
        with pytest.raises(smoe.MoeError) as e:
            smoe.moe_forward(h, layer.x, y, wait_limit_ns=200_000,
                             flags=smoe.MOE_FLAG_SYNC_CHECK | smoe.MOE_FLAG_TEST_STALL)
        assert e.value.status == smoe.MOE_ERR_TIMEOUT, e.value
        assert smoe.moe_get_device_status(h) == 0
        for _ in range(2):
            r = gu.run(smoe, h, layer)
            gu.check(gu.compare(layer, r.y, r.ids, r.w), fmt)
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)
