"""Host-side checks of the C-ABI library (no GPU needed): it loads, it
exports every function include/moe.h declares, status strings, and config
validation that happens before any device call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[\w]+\**\s+\**(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def smoe():
    import __graft_entry__
    __graft_entry__.build()
    import sparse_moe_sigmoid_b200 as m
    return m


def test_library_exports_every_declared_function(smoe):
    declared = _declared_functions()
    assert len(declared) >= 12, declared
    lib = ctypes.CDLL(smoe.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(smoe.EXPORTED)


def test_status_strings(smoe):
    assert smoe.moe_status_string(smoe.MOE_OK) == "ok"
    assert "unsupported" in smoe.moe_status_string(smoe.MOE_ERR_UNSUPPORTED)
    assert smoe.moe_status_string(12345) == "unknown status"


def test_config_defaults_are_k2(smoe):
    c = smoe.moe_config_init_k2()
    assert (c.hidden_size, c.moe_intermediate_size, c.n_routed_experts, c.num_experts_per_tok,
            c.n_shared_experts, c.n_group, c.topk_group, c.norm_topk_prob) == (
        7168, 2048, 384, 8, 1, 1, 1, 1)
    assert abs(c.routed_scaling_factor - 2.827) < 1e-6
    assert list(c.weight_block_size) == [128, 128]


@pytest.mark.parametrize("field,value,expect", [
    ("n_group", 64, "MOE_ERR_UNSUPPORTED"),       # more groups than warp lanes
    ("n_group", 5, "MOE_ERR_INVALID_ARG"),        # 384 experts do not split into 5 groups
    ("n_group", 0, "MOE_ERR_INVALID_ARG"),
    ("topk_group", 4, "MOE_ERR_INVALID_ARG"),     # more kept groups than groups (n_group 1)
    ("hidden_size", 7000, "MOE_ERR_UNSUPPORTED"),
    ("moe_intermediate_size", 100, "MOE_ERR_UNSUPPORTED"),
    ("n_routed_experts", 1024, "MOE_ERR_UNSUPPORTED"),
    ("num_experts_per_tok", 400, "MOE_ERR_INVALID_ARG"),
    ("max_tokens", 0, "MOE_ERR_INVALID_ARG"),
    ("scoring_func", 1, "MOE_ERR_UNSUPPORTED"),
    ("weight_block_size", (64, 128), None),
])
def test_create_rejects_bad_configs_before_touching_a_device(smoe, field, value, expect):
    c = smoe.moe_config_init_k2()
    if field == "weight_block_size":
        c.weight_format = smoe.MOE_WEIGHT_FP8_E4M3_BLOCK
        c.weight_block_size[0], c.weight_block_size[1] = value
        expect = "MOE_ERR_UNSUPPORTED"
    else:
        setattr(c, field, value)
    with pytest.raises(smoe.MoeError) as ei:
        smoe.moe_create(c, 0)
    assert ei.value.status == getattr(smoe, expect)


def test_group_limited_configs_are_checked_before_touching_a_device(smoe):
    """n_group > 1: the kept groups must hold at least k experts (here 48
    groups of 8 with one kept cannot supply 9 experts)."""
    c = smoe.moe_config_init_k2(n_group=48, topk_group=1, num_experts_per_tok=9)
    with pytest.raises(smoe.MoeError) as ei:
        smoe.moe_create(c, 0)
    assert ei.value.status == smoe.MOE_ERR_UNSUPPORTED  # n_group > 32 comes first
    c = smoe.moe_config_init_k2(n_group=32, topk_group=1, num_experts_per_tok=13)
    with pytest.raises(smoe.MoeError) as ei:
        smoe.moe_create(c, 0)
    assert ei.value.status == smoe.MOE_ERR_INVALID_ARG  # 1 group of 12 < 13 experts


@pytest.mark.parametrize("E,k,ns,expect", [
    (0, 8, 9, "MOE_ERR_INVALID_ARG"),   # no routed experts, yet k > 0
    (0, 0, 0, "MOE_ERR_INVALID_ARG"),   # no routed and no shared experts: no layer
    (384, 0, 1, "MOE_ERR_INVALID_ARG"),  # routed experts need k >= 1
    (0, 0, 17, "MOE_ERR_UNSUPPORTED"),  # shared MLP wider than 16 x f
])
def test_dense_layer_configs_are_checked_before_touching_a_device(smoe, E, k, ns, expect):
    """n_routed_experts = 0 (a dense FFN: the shared MLP alone) is a valid
    layer only with num_experts_per_tok = 0 and 1..16 shared groups."""
    c = smoe.moe_config_init_k2(n_routed_experts=E, num_experts_per_tok=k, n_shared_experts=ns)
    with pytest.raises(smoe.MoeError) as ei:
        smoe.moe_create(c, 0)
    assert ei.value.status == getattr(smoe, expect)


def test_null_handle_calls_are_rejected(smoe):
    lib = ctypes.CDLL(smoe.LIB_PATH)
    lib.moe_forward.restype = ctypes.c_int
    lib.moe_forward.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] + [ctypes.c_void_p] * 3
    assert lib.moe_forward(None, None, None, 4, None, None, None) == smoe.MOE_ERR_INVALID_ARG
    assert smoe.moe_launch_count(None) == 0
    smoe.moe_destroy(None)
