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
    r = _GOOD_ROUTE(x, router_weight, bias, k, routed_scaling_factor, norm_topk_prob, n_group,
                    topk_group)
    sel = np.take_along_axis(r.keys.astype(np.float64), r.ids, axis=1)  # biased keys as weights
    r.weights = sel / sel.sum(axis=1, keepdims=True) * routed_scaling_factor
    return r


def _bad_route_no_norm(x, router_weight, bias, k, routed_scaling_factor=2.827,
                       norm_topk_prob=True, n_group=1, topk_group=1):
    return _GOOD_ROUTE(x, router_weight, bias, k, routed_scaling_factor, False, n_group,
                       topk_group)


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
_GOOD_GROUP_FILTER = orc.group_filter
_GOOD_COMBINE_SUM = orc.combine


def _bad_group_score_max(keys, n_group, topk_group):
    # planted: a group scores its largest key only
    keys = np.asarray(keys, np.float32)
    T, E = keys.shape
    gs = E // n_group
    g = keys.reshape(T, n_group, gs).max(axis=2)
    order = np.argsort(-g.astype(np.float64), axis=1, kind="stable")
    kept = np.zeros((T, n_group), bool)
    np.put_along_axis(kept, order[:, :topk_group], True, axis=1)
    masked = np.where(np.repeat(kept, gs, axis=1), keys, np.float32(-np.inf)).astype(np.float32)
    return masked, np.full(T, np.inf)


def _bad_group_strided(keys, n_group, topk_group):
    # planted: group g holds the experts e with e % n_group == g
    keys = np.asarray(keys, np.float32)
    T, E = keys.shape
    perm = np.argsort(np.arange(E) % n_group, kind="stable")
    inv = np.argsort(perm)
    masked, gm = _GOOD_GROUP_FILTER(keys[:, perm], n_group, topk_group)
    return masked[:, inv], gm


def _bad_group_ties_high(keys, n_group, topk_group):
    # planted: equal group scores keep the higher group
    keys = np.asarray(keys, np.float32)
    T, E = keys.shape
    rev = np.arange(E).reshape(n_group, E // n_group)[::-1].ravel()
    masked, gm = _GOOD_GROUP_FILTER(keys[:, rev], n_group, topk_group)
    return masked[:, np.argsort(rev)], gm


def _bad_routing_weights_unnormalised(scores, ids, routed_scaling_factor=2.827,
                                      norm_topk_prob=True):
    sel = np.take_along_axis(np.asarray(scores, np.float64), np.asarray(ids, np.int64), axis=1)
    return sel * routed_scaling_factor


def _bad_combine_shared_scaled(pair_out, weights, shared_out=None):
    return _GOOD_COMBINE_SUM(pair_out, weights,
                             None if shared_out is None else 2.827 * shared_out)

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
    "group_score_max_key": ("group_filter", _bad_group_score_max),
    "group_strided": ("group_filter", _bad_group_strided),
    "group_ties_to_higher": ("group_filter", _bad_group_ties_high),
    "routing_weights_unnormalised": ("routing_weights", _bad_routing_weights_unnormalised),
    "combine_shared_scaled": ("combine", _bad_combine_shared_scaled),
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
