"""The dense FFN layer: K2's first layer ("Behind Kimi-K2's Config" §2.3,
first_k_dense = 1; "Kimi K2 Base" raw config: first_k_dense_replace 1,
intermediate_size 18432) is one SwiGLU MLP with no router. The library runs it
as a layer with n_routed_experts = 0 whose shared MLP, intermediate
9 x 2048 = 18432, is split into 9 groups of 2048 (an exact split of the down
projection's sum). Compared with the oracle's dense_ffn on the same matrices:
max|gpu - oracle| / max|oracle| <= 1e-2 (BF16) and <= 3e-2 (FP8), on every
token for the small layer and on a seeded sample at K2 sizes."""
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


def _dense_shape(d, f, ns):
    return synth.LayerShape(hidden_size=d, moe_intermediate_size=f, n_routed_experts=0,
                            num_experts_per_tok=0, n_shared_experts=ns)


def _run_dense(smoe, shape, fmt, T, tokens=None):
    x = synth.make_tokens(shape, T, device="cuda")
    ew = synth.make_experts(shape, device="cuda", fmt=fmt)
    cfg = smoe.moe_config_init_k2(
        hidden_size=shape.hidden_size, moe_intermediate_size=shape.moe_intermediate_size,
        n_routed_experts=0, num_experts_per_tok=0, n_shared_experts=shape.n_shared_experts,
        max_tokens=T,
        weight_format=smoe.MOE_WEIGHT_BF16 if fmt == "bf16" else smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    h = smoe.moe_create(cfg, 0)
    try:
        # the router and routed-expert weights are absent (NULL)
        smoe.moe_load_weights(h, None, None, None, None, None, ew.shared_gate, ew.shared_up,
                              ew.shared_down, shared_gate_scale=ew.shared_gate_scale,
                              shared_up_scale=ew.shared_up_scale,
                              shared_down_scale=ew.shared_down_scale)
        y = torch.empty_like(x)
        n0 = smoe.moe_launch_count(h)
        smoe.moe_forward(h, x, y, flags=smoe.MOE_FLAG_SYNC_CHECK)
        launches = smoe.moe_launch_count(h) - n0
    finally:
        smoe.moe_destroy(h)
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    mats = {n: gu.f64(v) for n, v in synth.shared_slice(ew).items()}
    del ew
    yo = orc.dense_ffn(gu.f64(x)[toks], mats, fmt)
    yg = gu.to_np(y).astype(np.float64)[toks]
    return float(np.max(np.abs(yg - yo)) / np.max(np.abs(yo))), launches


@pytest.mark.parametrize("fmt,T", [("bf16", 1), ("bf16", 37), ("bf16", 300), ("fp8", 1),
                                   ("fp8", 64), ("fp8", 200)])
def test_small_dense_ffn(smoe, fmt, T):
    """d = 256, intermediate 3 x 128 = 384: every token."""
    err, launches = _run_dense(smoe, _dense_shape(256, 128, 3), fmt, T)
    assert err <= gu.TOL[fmt], err
    # no router: scan, dispatch, gate/up, down, combine
    assert launches == 5


@pytest.mark.parametrize("fmt,T", [("bf16", 64), ("bf16", 2048), ("fp8", 64), ("fp8", 1024)])
def test_k2_dense_ffn(smoe, fmt, T):
    """K2's dense layer: d = 7168, intermediate 9 x 2048 = 18432 (T = 2048 runs
    the CTA-pair BF16 kernels, T = 64 the one-SM ones); every token at T = 64,
    512 sampled tokens (the first and last among them) otherwise."""
    toks = gu.sample_tokens(T)
    err, _ = _run_dense(smoe, _dense_shape(7168, 2048, 9), fmt, T, toks)
    print(f"dense {fmt} T={T}: {len(toks)} tokens, max rel err {err:.2e}")
    assert err <= gu.TOL[fmt], err


@pytest.mark.parametrize("fmt", ["bf16", "fp8"])
def test_dense_ffn_odd_sizes(smoe, fmt):
    """d = 384 and intermediate 2 x 384 (odd multiples of 128: no 256-feature
    down tiles, no CTA pairs): every token."""
    err, launches = _run_dense(smoe, _dense_shape(384, 384, 2), fmt, 100)
    assert err <= gu.TOL[fmt], err
    assert launches == 5
