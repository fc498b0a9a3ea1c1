"""moe_router_topk_noalloc: the router for callers that cannot allocate device
memory (an engine whose memory pool owns the GPU, or a step that cannot take
cudaMalloc's synchronisation). Its scratch is a static device array in the
library, so it takes no handle.

Checked through the C ABI against the oracle's routing (sets exact except
near-ties, which must stay valid; weights to 1e-5 against the oracle's
weights for the chosen experts) and against moe_forward's routing of the same
tokens, on calls in a row with different token counts, so that each call runs
on the array the previous one left behind. The token counts cover the three
routers moe_forward picks from (a GEMV for T <= 8, the split-K kernel this
entry point always uses, the tensor-core router for T >= 512): where they sum
in another order, only near-tie tokens may choose differently.

This file is named to be collected last: it must pass alone in a fresh
process and after every other test.
"""
import numpy as np
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_noalloc_router_matches_oracle_and_forward():
    import sparse_moe_sigmoid_b200 as smoe
    # K2 router sizes (7168 x 384, top-8) with small experts to keep the layer cheap
    shape = synth.LayerShape(moe_intermediate_size=128)
    layer = gu.make_layer(shape, 1024, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=1024)
    r = gu.oracle_route(layer)
    try:
        for T in (300, 5, 1024, 64):
            x = layer.x[:T].contiguous()
            # the phase kernels: their router at 8 < T < 512 is this entry point's
            fwd = gu.run(smoe, h, layer, x, flags=smoe.MOE_FLAG_PHASE_KERNELS)
            ids = torch.full((T, 8), -1, dtype=torch.int32, device="cuda")
            w = torch.zeros((T, 8), dtype=torch.float32, device="cuda")
            smoe.moe_router_topk_noalloc(x, layer.Wg, layer.b, 8, ids, w)
            torch.cuda.synchronize()
            gid = gu.to_np(ids).astype(np.int64)
            rc = gu.check_routing(r, gid, gu.to_np(w).astype(np.float64), 384, 2.827, True)
            print(f"T={T}: near-ties {int(rc.tie.sum())}, "
                  f"{int(np.sum(~rc.same_set & rc.tie))} chose the other side")
            assert rc.mismatch == 0 and rc.invalid == 0, T
            assert rc.weight_max_rel < 1e-5, (T, rc.weight_max_rel)
            np.testing.assert_allclose(gu.to_np(w).sum(axis=1), 2.827, rtol=1e-5)
            # against moe_forward: the same sets except where the oracle's
            # keys are near-tied; identical where both use the split-K router
            same = np.array([set(a) == set(b) for a, b in zip(gid, gu.to_np(fwd.ids))])
            assert np.all(same | rc.tie), T
            if 8 < T < 512:
                assert torch.equal(ids, fwd.ids), T
                assert torch.equal(w, fwd.w), T
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)


def test_noalloc_router_rejects_sizes_beyond_its_scratch():
    import sparse_moe_sigmoid_b200 as smoe
    E, d, T = 384, 256, 12000  # T * E * 4 bytes of partial logits alone exceed 16 MiB
    x = torch.zeros((T, d), dtype=torch.bfloat16, device="cuda")
    Wg = torch.zeros((E, d), dtype=torch.float32, device="cuda")
    b = torch.zeros((E,), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, 8), dtype=torch.int32, device="cuda")
    w = torch.empty((T, 8), dtype=torch.float32, device="cuda")
    with pytest.raises(smoe.MoeError) as e:
        smoe.moe_router_topk_noalloc(x, Wg, b, 8, ids, w)
    assert e.value.status == smoe.MOE_ERR_INVALID_ARG
    # a token count far past the array (the size arithmetic must not wrap)
    with pytest.raises(smoe.MoeError) as e:
        smoe.moe_router_topk_noalloc(x, Wg, b, 8, ids, w, T=1 << 62)
    assert e.value.status == smoe.MOE_ERR_INVALID_ARG
