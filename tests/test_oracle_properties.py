"""Randomised properties of the oracle's router (sigmoid scores, noaux_tc
biased top-k, normalise, scale: the "Kimi K2 Base" raw config fields
scoring_func sigmoid, topk_method noaux_tc, norm_topk_prob true,
routed_scaling_factor 2.827) and of its combine, over many small shapes.

Inputs are drawn on coarse grids so that equal keys occur often and the
tie rule (equal keys: lower expert index first) is exercised. These add
breadth to the fixed-seed pins; they do not restate the formulas."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import moe as orc

SETTINGS = settings(max_examples=60, deadline=None)


@st.composite
def router_case(draw):
    T = draw(st.integers(1, 5))
    E = draw(st.integers(2, 20))
    k = draw(st.integers(1, E))
    d = draw(st.integers(1, 8))
    seed = draw(st.integers(0, 2**32 - 1))
    rng = np.random.default_rng(seed)
    # quarter-integer grids: many exactly equal logits, scores and keys
    x = rng.integers(-4, 5, (T, d)) / 4.0
    W = rng.integers(-2, 3, (E, d)) / 4.0
    bias = rng.integers(-2, 3, E) / 8.0
    return x, W, bias, k


def _keys(x, W, bias):
    return orc.selection_keys(orc.router_logits(x, W), bias).astype(np.float64)


@SETTINGS
@given(router_case())
def test_selection_is_a_valid_topk_with_the_tie_rule(case):
    x, W, bias, k = case
    r = orc.route(x, W, bias, k)
    keys = _keys(x, W, bias)
    E = W.shape[0]
    for t in range(x.shape[0]):
        ids = r.ids[t]
        assert len(set(ids.tolist())) == k and ids.min() >= 0 and ids.max() < E
        rest = np.setdiff1d(np.arange(E), ids)
        for e in rest:  # nothing left out beats anything chosen, ties to the lower index
            for j in ids:
                assert keys[t, j] > keys[t, e] or (keys[t, j] == keys[t, e] and j < e)
        for a, b in zip(ids[:-1], ids[1:]):  # slots: key descending, equal keys by index
            assert keys[t, a] > keys[t, b] or (keys[t, a] == keys[t, b] and a < b)


@SETTINGS
@given(router_case())
def test_weights_are_positive_and_sum_to_the_scaling_factor(case):
    x, W, bias, k = case
    r = orc.route(x, W, bias, k)
    assert np.all(r.weights > 0)
    np.testing.assert_allclose(r.weights.sum(axis=1), 2.827, rtol=1e-12)
    raw = orc.route(x, W, bias, k, norm_topk_prob=False, routed_scaling_factor=1.0)
    # without normalisation the weights are the chosen unbiased sigmoid scores
    np.testing.assert_array_equal(raw.ids, r.ids)
    assert np.all((raw.weights > 0) & (raw.weights < 1))


@SETTINGS
@given(router_case(), st.sampled_from([-0.5, -0.125, 0.25, 1.0]))
def test_a_uniform_bias_shift_changes_nothing(case, c):
    # exact in float32 for these grid values: every key moves by the same c
    x, W, bias, k = case
    a = orc.route(x, W, bias, k)
    b = orc.route(x, W, bias + c, k)
    np.testing.assert_array_equal(a.ids, b.ids)
    np.testing.assert_array_equal(a.weights, b.weights)


@SETTINGS
@given(router_case(), st.integers(0, 2**32 - 1))
def test_relabelling_the_experts_relabels_the_choice(case, pseed):
    x, W, bias, k = case
    E = W.shape[0]
    perm = np.random.default_rng(pseed).permutation(E)  # new expert i is old perm[i]
    a = orc.route(x, W, bias, k)
    b = orc.route(x, W[perm], bias[perm], k)
    keys = _keys(x, W, bias)
    for t in range(x.shape[0]):
        ka = np.sort(keys[t, a.ids[t]])
        kb = np.sort(keys[t, perm[b.ids[t]]])
        np.testing.assert_array_equal(ka, kb)  # the same chosen key values
        if a.margin[t] > 0:  # no tie at the cut: the same experts, same weights
            assert set(a.ids[t].tolist()) == set(perm[b.ids[t]].tolist())
            wa = dict(zip(a.ids[t].tolist(), a.weights[t]))
            for j, w in zip(perm[b.ids[t]].tolist(), b.weights[t]):
                np.testing.assert_allclose(w, wa[j], rtol=1e-12)


@SETTINGS
@given(router_case())
def test_each_token_is_routed_on_its_own(case):
    x, W, bias, k = case
    r = orc.route(x, W, bias, k)
    for t in range(x.shape[0]):
        one = orc.route(x[t:t + 1], W, bias, k)
        np.testing.assert_array_equal(one.ids[0], r.ids[t])
        np.testing.assert_allclose(one.weights[0], r.weights[t], rtol=1e-12)


@settings(max_examples=25, deadline=None)
@given(st.integers(0, 2**32 - 1))
def test_combine_adds_the_shared_expert_and_is_linear_in_the_weights(seed):
    rng = np.random.default_rng(seed)
    T, d, f, E, k = 3, 6, 5, 4, 2
    x = rng.standard_normal((T, d))
    mats = [{"gate": rng.standard_normal((f, d)), "up": rng.standard_normal((f, d)),
             "down": rng.standard_normal((d, f))} for _ in range(E + 1)]
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    w = rng.random((T, k)) + 0.1
    get = lambda e: mats[e]
    routed = orc.experts_combine(x, ids, w, get, None)
    full = orc.experts_combine(x, ids, w, get, lambda: mats[E])
    shared = orc.experts_combine(x, np.zeros((T, 0), np.int64), np.zeros((T, 0)), None,
                                 lambda: mats[E])
    np.testing.assert_allclose(full, routed + shared, rtol=1e-12, atol=1e-12)
    # the shared expert enters with weight 1: as a routed expert chosen with weight 1
    as_routed = orc.experts_combine(x, np.full((T, 1), E), np.ones((T, 1)), get, None)
    np.testing.assert_allclose(shared, as_routed, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(orc.experts_combine(x, ids, 3.0 * w, get, None), 3.0 * routed,
                               rtol=1e-12, atol=1e-12)
