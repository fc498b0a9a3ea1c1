"""moe_router_topk_noalloc: the router for callers that cannot allocate device
memory (an engine whose memory pool owns the GPU, or a step that cannot take
cudaMalloc's synchronisation). Its scratch is a static device array in the
library, so it takes no handle.

Checked through the C ABI against the routing that moe_forward reports for
the same inputs (topk_ids_out / topk_weights_out), on two calls in a row with
different token counts, so the second call runs on the array the first one
left behind. Both paths use the same kernels and split count here, so the
expert ids must match exactly and the weights to the tests' 1e-5.

This file is named to be collected last: it must pass alone in a fresh
process and after every other test.
"""
import pytest
import torch

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


def test_noalloc_router_matches_forward_routing_twice():
    import sparse_moe_sigmoid_b200 as smoe
    # K2 router sizes (7168 x 384, top-8) with small experts to keep the layer cheap
    shape = synth.LayerShape(moe_intermediate_size=128)
    layer = gu.make_layer(shape, 300, "bf16")
    h = gu.create_handle(smoe, layer, max_tokens=300)
    try:
        for T in (300, 64):
            x = layer.x[:T].contiguous()
            _, ids_ref, w_ref = gu.run(smoe, h, layer, x)
            ids = torch.full((T, 8), -1, dtype=torch.int32, device="cuda")
            w = torch.zeros((T, 8), dtype=torch.float32, device="cuda")
            smoe.moe_router_topk_noalloc(x, layer.Wg, layer.b, 8, ids, w)
            torch.cuda.synchronize()
            assert torch.equal(ids, ids_ref), T
            torch.testing.assert_close(w, w_ref, rtol=1e-5, atol=0)
            assert torch.allclose(w.sum(dim=1), torch.full((T,), 2.827, device="cuda"), rtol=1e-5)
    finally:
        smoe.moe_destroy(h)


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
