"""Expert parallelism through the library on one GPU (world size 1, NCCL):
every piece an EP rank runs on its GPU — the router over all experts, its
slice of the experts with the expert forced per row, the shared expert as a
dense layer, the exchange, and the combine of the returned rows — against the
oracle, and moe_combine_rows alone against the oracle's combine. The
exchange between several GPUs is tested on CPU ranks (tests/test_ep_host.py);
nothing here needs more than one GPU."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
from oracle import moe as orc
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


@pytest.fixture(scope="module")
def nccl_world1():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


def test_combine_rows_matches_the_oracle(smoe):
    g = torch.Generator(device="cuda").manual_seed(4)
    T, k, d = 37, 4, 512
    pair = torch.randn((T * k, d), generator=g, device="cuda").to(torch.bfloat16)
    shared = torch.randn((T, d), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.rand((T, k), generator=g, device="cuda")
    y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    smoe.moe_combine_rows(pair, w, shared, y)
    torch.cuda.synchronize()
    want = orc.combine(gu.f64(pair).reshape(T, k, d), gu.f64(w), gu.f64(shared))
    err = np.max(np.abs(gu.f64(y) - want)) / np.max(np.abs(want))
    assert err <= 2 ** -8, err  # one BF16 rounding of an fp32 sum
    y0 = torch.empty_like(y)
    smoe.moe_combine_rows(pair, w, None, y0)  # no shared expert
    want0 = orc.combine(gu.f64(pair).reshape(T, k, d), gu.f64(w), None)
    assert np.max(np.abs(gu.f64(y0) - want0)) / np.max(np.abs(want0)) <= 2 ** -8


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
@pytest.mark.parametrize("T", [1, 40, 300])
def test_ep_rank_on_one_gpu_matches_the_oracle(smoe, nccl_world1, fmt, T):
    from sparse_moe_sigmoid_b200 import ep
    layer = gu.make_layer(synth.TINY, 300, fmt)
    cfg = smoe.moe_config_init_k2(
        hidden_size=256, moe_intermediate_size=128, n_routed_experts=16, num_experts_per_tok=4,
        n_shared_experts=1,
        weight_format=smoe.MOE_WEIGHT_BF16 if fmt == "bf16" else smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    ew = layer.ew
    L = ep.LibraryEP(smoe, cfg, layer.Wg, layer.b, ew.gate, ew.up, ew.down, ew.shared_gate,
                     ew.shared_up, ew.shared_down, max_tokens=300,
                     gate_scale=ew.gate_scale, up_scale=ew.up_scale, down_scale=ew.down_scale,
                     shared_gate_scale=ew.shared_gate_scale, shared_up_scale=ew.shared_up_scale,
                     shared_down_scale=ew.shared_down_scale)
    try:
        x = layer.x[:T].contiguous()
        ids, w = L.route(x)
        y = L.forward(x)
        torch.cuda.synchronize()
    finally:
        L.close()
    rep = gu.compare(layer, y, ids, w, x=x)
    gu.check(rep, fmt)
    gu.release(layer)
