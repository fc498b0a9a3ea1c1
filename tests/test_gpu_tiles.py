"""Every row-tile height the planner can pick, on the GPU against the oracle.

The row tile is the smallest supported height >= 3 x the mean rows per routed
expert (BF16: 16, 32, 64, 96, 128, 160, 192, 224, 256; FP8 gate/up: 16, 32,
64, 96; FP8 down: 16, 32, 64, 128, 192). With 8 experts and top-2 the mean is
T / 4, so the token counts below land on each height in turn (and T = 1200
on the tallest with several tiles per expert). Two layer shapes take the
different kernel paths: d = 384 (an odd multiple of 128: one 128-row weight
tile per down unit, no CTA pairs) and d = 512 with f = 256 (256-feature down
units, CTA pairs from 128 rows in BF16). Outputs of up to 512 tokens each
are compared with the oracle, with the acceptance rule of the other parity
tests.
"""
import pytest

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

SHAPES = {"d384": synth.LayerShape(384, 128, 8, 2, 1),
          "d512_f256": synth.LayerShape(512, 256, 8, 2, 1)}
# T -> tile height (3 T / 4 rounded up to the next supported height)
T_BF16 = [16, 40, 84, 124, 168, 212, 252, 296, 340, 1200]
T_FP8 = [16, 40, 84, 124, 168, 252, 1200]
CASES = [(s, "bf16", T) for s in SHAPES for T in T_BF16] + \
        [(s, "fp8", T) for s in SHAPES for T in T_FP8]


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


@pytest.fixture(scope="module")
def layers():
    made = {}
    yield made
    for layer in made.values():
        gu.release(layer)


@pytest.mark.parametrize("shape,fmt,T", CASES, ids=[f"{s}-{f}-T{T}" for s, f, T in CASES])
def test_tile_height_matches_the_oracle(smoe, layers, shape, fmt, T):
    key = (shape, fmt)
    if key not in layers:
        layers[key] = gu.make_layer(SHAPES[shape], max(T_BF16), fmt)
    layer = layers[key]
    h = gu.create_handle(smoe, layer, max_tokens=T)
    try:
        x = layer.x[:T].contiguous()
        r = gu.run(smoe, h, layer, x)
        gu.check(gu.compare(layer, r.y, r.ids, r.w, x=x), fmt)
    finally:
        smoe.moe_destroy(h)
