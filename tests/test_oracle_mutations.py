"""Plant plausible mistakes in the oracle (on the CPU) and check that at least
one pin catches each of them. A pin that lets a planted mistake through
would also let a real one through."""
import numpy as np
import pytest

from oracle import e4m3 as e4
from oracle import moe as orc
from tests import pins


def _bad_route_weights_from_keys(x, router_weight, bias, k, routed_scaling_factor=2.827,
                                 norm_topk_prob=True, n_group=1, topk_group=1):
    logits = orc.router_logits(x, router_weight)
    keys = orc.selection_keys(logits, bias)
    ids, margin = orc.topk_by_key(keys, k)
    sel = np.take_along_axis(keys.astype(np.float64), ids, axis=1)  # biased keys as weights
    w = sel / sel.sum(axis=1, keepdims=True) * routed_scaling_factor
    return orc.Routing(ids, w, orc.sigmoid(logits), keys, margin)


def _bad_route_no_norm(x, router_weight, bias, k, routed_scaling_factor=2.827,
                       norm_topk_prob=True, n_group=1, topk_group=1):
    r = _GOOD_ROUTE(x, router_weight, bias, k, routed_scaling_factor, False)
    return r


def _bad_topk_ascending(key, k):
    order = np.argsort(key, axis=1, kind="stable")
    return order[:, :k].astype(np.int64), np.ones(key.shape[0])


def _bad_sigmoid(z):
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(z))


def _bad_swiglu_swapped(xr, w_gate, w_up, w_down):
    return _GOOD_SWIGLU(xr, w_up, w_gate, w_down)


def _bad_silu_no_gate(z):
    return np.asarray(z, np.float64)


def _bad_act_quant_scale(v, group=128):
    v = np.asarray(v, np.float32)
    n, c = v.shape
    vg = v.reshape(n, c // group, group)
    amax = np.abs(vg).max(axis=2)
    s = np.where(amax == 0, 1.0, amax / 240.0).astype(np.float32)  # wrong full-scale value
    codes = e4.encode((vg / s[:, :, None]).astype(np.float64)).reshape(n, c)
    return codes, s


def _bad_weight_dequant_transposed_blocks(codes, scales, block=128):
    return _GOOD_WDQ(codes, np.ascontiguousarray(np.asarray(scales)[::-1, ::-1]), block)


def _bad_expert_params(d, f):
    return 2 * d * f


_GOOD_ROUTE = orc.route
_GOOD_SWIGLU = orc.swiglu_expert
_GOOD_WDQ = orc.weight_dequant


def _shared_scaled_combine(x, ids, weights, get_expert, get_shared, fmt="bf16",
                           n_shared_experts=1, tokens=None):
    # planted: the shared expert is multiplied by the routed scaling factor
    y = _GOOD_COMBINE(x, ids, weights, get_expert, None, fmt, n_shared_experts, tokens)
    if get_shared is not None:
        m = get_shared()
        xs = np.asarray(x, np.float64) if tokens is None else np.asarray(x, np.float64)[tokens]
        y = y + 2.827 * _GOOD_SWIGLU(xs, m["gate"], m["up"], m["down"])
    return y


_GOOD_COMBINE = orc.experts_combine

MUTATIONS = {
    "weights_from_biased_keys": ("route", _bad_route_weights_from_keys),
    "no_normalisation": ("route", _bad_route_no_norm),
    "topk_ascending": ("topk_by_key", _bad_topk_ascending),
    "sigmoid_sign": ("sigmoid", _bad_sigmoid),
    "gate_up_swapped": ("swiglu_expert", _bad_swiglu_swapped),
    "silu_without_gate": ("silu", _bad_silu_no_gate),
    "shared_scaled": ("experts_combine", _shared_scaled_combine),
    "act_quant_wrong_scale": ("act_quant", _bad_act_quant_scale),
    "weight_scale_misindexed": ("weight_dequant", _bad_weight_dequant_transposed_blocks),
    "expert_params_two_mats": ("expert_params", _bad_expert_params),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(orc, attr, bad)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"planted mistake {name} passed every pin"


def test_e4m3_bias_mutation_is_caught(monkeypatch):
    bad = np.array([e4.decode_scalar(c) * 2.0 for c in range(256)])  # exponent bias 6
    monkeypatch.setattr(e4, "_DECODE_TABLE", bad)
    import tests.test_oracle_e4m3 as t
    with pytest.raises(AssertionError):
        t.test_decode_all_codes_match_torch()
