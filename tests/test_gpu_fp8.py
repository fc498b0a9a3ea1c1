"""FP8 path (e4m3 weights with 128x128 block scales, dynamic per-token
per-128-column activation quantisation) against the oracle.

The activation quantisation is integer output (codes) decided in fp32 on
both sides, so it must be bit-exact. Layer outputs: max|gpu - oracle| /
max|oracle| <= 3e-2, the oracle applying the same block dequantisation and
the same activation quantisation (of its own float64 h rounded to fp32).
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


def test_activation_quant_is_bit_exact(smoe):
    g = torch.Generator(device="cuda").manual_seed(3)
    rows, cols = 97, 7168
    x = torch.randn((rows, cols), generator=g, device="cuda")
    scale = torch.tensor([1e-6, 1e-3, 1.0, 30.0, 1e4], device="cuda")
    x = (x * scale[torch.arange(rows, device="cuda") % 5].unsqueeze(1)).to(torch.bfloat16)
    x[5, 256:384] = 0  # an all-zero group: scale 1, codes 0
    x[7, 0] = 3.0e38   # a huge value: the rest of its group underflows to code 0
    q = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, cols // 128), dtype=torch.float32, device="cuda")
    smoe.moe_act_quant_e4m3(x, q, s)
    torch.cuda.synchronize()
    codes, scales = orc.act_quant(x.float().cpu().numpy())
    assert np.array_equal(s.cpu().numpy(), scales)
    assert np.array_equal(q.cpu().numpy(), codes)


@pytest.fixture(scope="module")
def tiny8(smoe):
    layer = gu.make_layer(synth.TINY, 256, "fp8")
    h = gu.create_handle(smoe, layer, max_tokens=256)
    yield layer, h
    smoe.moe_destroy(h)
    gu.release(layer)


def _check(rep, **kw):
    gu.check(rep, "fp8", **kw)


@pytest.mark.parametrize("T", [1, 5, 64, 200, 256])
def test_tiny_fp8(smoe, tiny8, T):
    layer, h = tiny8
    x = layer.x[:T].contiguous()
    y, ids, w = gu.run(smoe, h, layer, x)
    _check(gu.compare(layer, y, ids, w, x=x))


def test_tiny_fp8_forced_routing(smoe, tiny8):
    layer, h = tiny8
    r = gu.oracle_route(layer)
    forced = torch.from_numpy(r.ids.astype(np.int32)).cuda()
    y, ids, _ = gu.run(smoe, h, layer, forced=forced)
    yo = gu.oracle_outputs(layer, r.ids, r.weights, np.arange(layer.x.shape[0]))
    err = np.max(np.abs(gu.to_np(y) - yo)) / np.max(np.abs(yo))
    assert err <= gu.TOL["fp8"]


def test_fp8_on_grid_matches_bf16(smoe):
    """Weights on the e4m3 grid with power-of-two block scales and x on the
    e4m3 grid with each group's largest value 448 * 2^-7: the BF16 layer
    holds exactly the same weight values and x quantises losslessly, so the
    FP8 output differs from the BF16 output only by h's e4m3 rounding
    (at most 2^-4 relative per element; bound used: 0.1)."""
    shape = synth.TINY
    l8 = gu.make_layer(shape, 64, "fp8")
    ew = l8.ew
    for n in ("gate_scale", "up_scale", "down_scale", "shared_gate_scale", "shared_up_scale",
              "shared_down_scale"):
        t = getattr(ew, n)
        t.copy_(torch.exp2(torch.round(torch.log2(t))))
    g = torch.Generator(device="cuda").manual_seed(9)
    codes = torch.randint(0, 0x7E, (64, shape.hidden_size), generator=g, device="cuda")
    codes |= torch.randint(0, 2, codes.shape, generator=g, device="cuda") * 0x80
    xg = codes.to(torch.uint8).view(torch.float8_e4m3fn).float()
    xg[:, ::128] = 448.0
    l8.x = (xg * 2.0 ** -7).to(torch.bfloat16)
    dec = lambda c: c.view(torch.float8_e4m3fn).float()

    def bf(c, sc):
        *lead, R, C = c.shape
        w = dec(c).reshape(*lead, R // 128, 128, C // 128, 128) * sc.unsqueeze(-2).unsqueeze(-1)
        return w.reshape(*lead, R, C).to(torch.bfloat16)

    ewb = synth.ExpertWeights("bf16", bf(ew.gate, ew.gate_scale), bf(ew.up, ew.up_scale),
                              bf(ew.down, ew.down_scale), bf(ew.shared_gate, ew.shared_gate_scale),
                              bf(ew.shared_up, ew.shared_up_scale),
                              bf(ew.shared_down, ew.shared_down_scale))
    lb = gu.Layer(shape, "bf16", l8.x, l8.Wg, l8.b, ewb)
    h8 = gu.create_handle(smoe, l8, 64)
    hb = gu.create_handle(smoe, lb, 64)
    try:
        y8, i8, _ = gu.run(smoe, h8, l8)
        yb, ib, _ = gu.run(smoe, hb, lb)
    finally:
        smoe.moe_destroy(h8)
        smoe.moe_destroy(hb)
    assert torch.equal(i8, ib)
    a, b = gu.to_np(y8), gu.to_np(yb)
    assert np.max(np.abs(a - b)) / np.max(np.abs(b)) <= 0.1


K2_FP8_T = (1, 16, 128, 1024, 4096, 8192, 16384)


@pytest.fixture(scope="module")
def k2fp8(smoe):
    layer = gu.make_layer(synth.K2, 16384, "fp8")
    h = gu.create_handle(smoe, layer, max_tokens=16384)
    # one expert-major oracle pass for every sweep point's sample and every
    # near-tie token (each token's output does not depend on T)
    toks = np.unique(np.concatenate([gu.sample_tokens(T) for T in K2_FP8_T]))
    gu.cache_of(layer).prepare(toks, with_ties_below=16384)
    yield layer, h
    smoe.moe_destroy(h)
    gu.release(layer)


# The FP8 sweep's token counts. T = 4096 and up reach the tallest FP8 row
# tiles (96 rows gate/up with three promotion warpgroups; 128 and 192 rows
# down). Routing is checked for every token; outputs on every token up to 512,
# else on 512 sampled tokens plus every near-tie token; the row order of
# every (token, slot) pair.
@pytest.mark.parametrize("T", K2_FP8_T)
def test_k2_fp8(smoe, k2fp8, T):
    layer, h = k2fp8
    x = layer.x[:T].contiguous()
    r = gu.run(smoe, h, layer, x, permutation=True)
    _check(gu.compare(layer, r.y, r.ids, r.w, x=x))
    print(gu.check_permutation(gu.to_np(r.ids), gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
