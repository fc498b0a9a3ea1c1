"""Layer shapes away from K2's, on the GPU against the oracle.

The library accepts any hidden_size and moe_intermediate_size that are
multiples of 128 (up to 16384 and 8192), up to 512 routed experts, top-k up
to 32 and up to 16 shared experts. Each case below is a fixed, seeded layer
chosen to reach a path the K2 shapes do not: sizes that are odd multiples of
128 (no 256-feature down tiles, no CTA pairs), a single or very few experts
(tall row tiles, FP8 promotion with three warpgroups), many experts, k = 1,
odd and maximal k, the longest FP8 K (64 blocks), group-limited routing in
FP8, unnormalised weights and other scaling factors, 16 shared groups, and
the single launch (the dense layer's odd sizes are in
test_gpu_dense.py). Every token's output is compared
(T <= 1000), with the acceptance rule of the other parity tests, and the
dispatch's row order is checked against the routing.
"""
import numpy as np
import pytest

import synth
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu

S = synth.LayerShape

# (name, shape, T, fmt, single_launch_max_tokens)
CASES = [
    ("d128_f128", S(128, 128, 8, 2, 1), 37, "bf16", 0),
    ("d384_f384_ns2", S(384, 384, 24, 6, 2), 200, "bf16", 0),
    ("d384_f256_ns0_fp8", S(384, 256, 24, 6, 0), 200, "fp8", 0),
    ("d512_f640_fp8", S(512, 640, 40, 8, 1), 333, "fp8", 0),
    ("three_experts_k1", S(1024, 256, 3, 1, 1), 1000, "bf16", 0),
    ("three_experts_f384", S(1024, 384, 3, 2, 0), 1000, "bf16", 0),
    ("k13_d2304", S(2304, 512, 100, 13, 1), 100, "bf16", 0),
    ("k32", S(256, 128, 64, 32, 0), 50, "bf16", 0),
    ("grouped_fp8", S(768, 256, 48, 8, 1, n_group=8, topk_group=3), 300, "fp8", 0),
    ("one_expert_fp8", S(1280, 1024, 1, 1, 1), 600, "fp8", 0),
    ("e512", S(512, 128, 512, 8, 1), 64, "bf16", 0),
    ("f8192_fp8", S(128, 8192, 4, 2, 1), 20, "fp8", 0),
    ("single_launch_bf16", S(512, 256, 24, 4, 1), 16, "bf16", 128),
    ("single_launch_fp8", S(512, 256, 24, 4, 1), 16, "fp8", 128),
    # routing settings other than K2's: weights not normalised, other scales
    ("no_norm_scale1", S(512, 256, 32, 6, 1, routed_scaling_factor=1.0, norm_topk_prob=False),
     200, "bf16", 0),
    ("no_norm_scale2p5_fp8", S(512, 256, 32, 6, 0, routed_scaling_factor=2.5,
                               norm_topk_prob=False), 200, "fp8", 0),
    ("grouped_top1", S(256, 128, 16, 1, 1, n_group=4, topk_group=1), 100, "bf16", 0),
    ("sixteen_shared", S(256, 128, 8, 2, 16), 50, "bf16", 0),
    ("single_launch_no_norm", S(512, 256, 24, 4, 1, norm_topk_prob=False), 16, "bf16", 128),
    ("single_launch_grouped_fp8", S(512, 256, 24, 4, 1, n_group=4, topk_group=2), 16, "fp8",
     128),
    # few tokens with fewer experts than the small-batch top-k's four warps
    ("three_experts_few_tokens", S(512, 256, 3, 2, 1), 100, "bf16", 0),
    ("one_expert_few_tokens", S(512, 256, 1, 1, 0), 50, "fp8", 0),
]


@pytest.fixture(scope="module")
def smoe():
    import sparse_moe_sigmoid_b200 as m
    return m


@pytest.mark.parametrize("name,shape,T,fmt,sl", CASES, ids=[c[0] for c in CASES])
def test_shape_matches_the_oracle(smoe, name, shape, T, fmt, sl):
    layer = gu.make_layer(shape, T, fmt)
    h = gu.create_handle(smoe, layer, max_tokens=T, single_launch_max_tokens=sl)
    try:
        n0 = smoe.moe_launch_count(h)
        r = gu.run(smoe, h, layer, permutation=True)
        if sl:
            assert smoe.moe_launch_count(h) - n0 == 1  # the whole layer in one launch
        rep = gu.compare(layer, r.y, r.ids, r.w, tokens=np.arange(T))
        gu.check(rep, fmt, min_compared=T)
        print(gu.check_permutation(gu.to_np(r.ids), gu.to_np(r.offsets), gu.to_np(r.pair_rows)))
    finally:
        smoe.moe_destroy(h)
        gu.release(layer)
