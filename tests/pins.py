"""Checks that pin the CPU oracle to facts fixed outside the oracle itself.

Each check takes the oracle module (oracle.moe) and raises AssertionError when
the oracle disagrees with: brute-force scalar loops (oracle.brute), a closed
form, an invariant the config fields imply, a textbook value, or a value the
pages print (tests/golden/). The same checks run against planted mistakes in
tests/test_oracle_mutations.py, which asserts that each mistake is caught.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import brute
from oracle import e4m3 as e4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _bf16_round(a):
    """Round float64 values to the nearest BF16 value (ties to even)."""
    a32 = np.asarray(a, np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def small_layer(seed, T, d, f, E, k, shared=True, wstd=0.2):
    """A random small layer (BF16-valued weights) as float64 arrays."""
    r = _rng(seed)
    x = _bf16_round(r.standard_normal((T, d)))
    Wg = r.standard_normal((E, d)).astype(np.float32).astype(np.float64) * 0.05
    b = (r.standard_normal(E) * 0.01).astype(np.float32).astype(np.float64)
    ex = [tuple(_bf16_round(r.standard_normal(s) * wstd) for s in ((f, d), (f, d), (d, f)))
          for _ in range(E)]
    sh = tuple(_bf16_round(r.standard_normal(s) * wstd) for s in ((f, d), (f, d), (d, f))) if shared else None
    return x, Wg, b, ex, sh


def _getters(ex, sh):
    ge = lambda e: {"gate": ex[e][0], "up": ex[e][1], "down": ex[e][2]}
    gs = (lambda: {"gate": sh[0], "up": sh[1], "down": sh[2]}) if sh is not None else None
    return ge, gs


# ----------------------------------------------------------------------------
def pin_route_vs_brute(orc):
    """Router ids and weights equal the scalar-loop router on random tokens."""
    x, Wg, b, _, _ = small_layer(11, T=6, d=40, f=8, E=12, k=4, shared=False)
    r = orc.route(x, Wg, b, 4, 2.827, True)
    for t in range(x.shape[0]):
        ids, w = brute.route_token(x[t], Wg, b, 4)
        assert list(r.ids[t]) == ids, (t, r.ids[t], ids)
        np.testing.assert_allclose(r.weights[t], w, rtol=1e-12, atol=0)


def pin_layer_vs_brute_bf16(orc):
    """Whole layer (routing, SwiGLU experts, weighted combine, shared expert)
    equals the scalar-loop layer; d != f so a transposed operand cannot pass."""
    T, d, f, E, k = 3, 24, 10, 6, 2
    x, Wg, b, ex, sh = small_layer(12, T, d, f, E, k)
    ge, gs = _getters(ex, sh)
    y, r = orc.forward(x, Wg, b, ge, gs, k, 2.827, True, "bf16", 1)
    for t in range(T):
        yb, ids, _ = brute.layer_token(x[t], Wg, b, ex, sh, k)
        assert list(r.ids[t]) == ids
        np.testing.assert_allclose(y[t], yb, rtol=1e-10, atol=1e-12)


def _dequant_scalar(codes, scales):
    R, C = codes.shape
    out = np.zeros((R, C))
    for i in range(R):
        for j in range(C):
            out[i, j] = e4.decode_scalar(int(codes[i, j])) * float(scales[i // 128, j // 128])
    return out


def fp8_small_layer(seed, T=2, d=256, f=128, E=4, k=2):
    r = _rng(seed)
    x = _bf16_round(r.standard_normal((T, d)))
    Wg = (r.standard_normal((E, d)) * 0.05).astype(np.float32).astype(np.float64)
    b = (r.standard_normal(E) * 0.01).astype(np.float32).astype(np.float64)

    def q(shape):
        codes = r.integers(0, 256, size=shape, dtype=np.int64).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x30  # no NaN codes in a checkpoint
        scales = (r.uniform(0.5, 2.0, size=(shape[0] // 128, shape[1] // 128)) * 1e-3).astype(np.float32)
        return codes, scales

    ex = []
    for _ in range(E + 1):
        (gc, gs), (uc, us), (dc, ds) = q((f, d)), q((f, d)), q((d, f))
        ex.append({"gate": gc, "gate_scale": gs, "up": uc, "up_scale": us,
                   "down": dc, "down_scale": ds})
    return x, Wg, b, ex[:E], ex[E]


def pin_layer_vs_brute_fp8(orc):
    """FP8 layer (block dequant, dynamic activation quant of x and h) equals
    the scalar-loop layer with the scalar e4m3 codec."""
    x, Wg, b, ex, sh = fp8_small_layer(13)
    k = 2
    y, r = orc.forward(x, Wg, b, lambda e: ex[e], lambda: sh, k, 2.827, True, "fp8", 1)
    exd = [tuple(_dequant_scalar(m[n], m[n + "_scale"]) for n in ("gate", "up", "down")) for m in ex]
    shd = tuple(_dequant_scalar(sh[n], sh[n + "_scale"]) for n in ("gate", "up", "down"))
    for t in range(x.shape[0]):
        yb, ids, _ = brute.layer_token(x[t], Wg, b, exd, shd, k, fp8=True)
        assert list(r.ids[t]) == ids
        np.testing.assert_allclose(y[t], yb, rtol=1e-9, atol=1e-12)


def pin_dense_ffn_vs_brute(orc):
    """The dense FFN (no router) equals the scalar-loop SwiGLU MLP, BF16 and
    FP8 (d != i so a transposed operand cannot pass), and the layer's combine
    with no routed experts (k = 0) and that MLP as its shared expert gives the
    same y."""
    T, d, i = 3, 24, 40
    x, _, _, _, sh = small_layer(21, T, d, i, 1, 1)
    mats = {"gate": sh[0], "up": sh[1], "down": sh[2]}
    y = orc.dense_ffn(x, mats, "bf16")
    for t in range(T):
        np.testing.assert_allclose(y[t], brute.expert_token(x[t], *sh), rtol=1e-10, atol=1e-12)
    yc = orc.experts_combine(x, np.zeros((T, 0), np.int64), np.zeros((T, 0)), None,
                             lambda: mats, "bf16", 1)
    np.testing.assert_array_equal(yc, y)
    x8, _, _, _, sh8 = fp8_small_layer(22, T=2, d=256, f=128, E=1, k=1)
    y8 = orc.dense_ffn(x8, sh8, "fp8")
    shd = tuple(_dequant_scalar(sh8[n], sh8[n + "_scale"]) for n in ("gate", "up", "down"))
    for t in range(2):
        np.testing.assert_allclose(y8[t], brute.expert_token(x8[t], *shd, fp8=True), rtol=1e-9,
                                   atol=1e-12)


def pin_weights_sum(orc):
    """norm_topk_prob then routed_scaling_factor: the k weights of every token
    are positive and sum to 2.827."""
    x, Wg, b, _, _ = small_layer(14, T=64, d=96, f=8, E=64, k=8, shared=False)
    r = orc.route(x, Wg, b, 8, 2.827, True)
    assert np.all(r.weights > 0)
    np.testing.assert_allclose(r.weights.sum(axis=1), 2.827, rtol=1e-12)
    assert all(len(set(row)) == 8 for row in r.ids.tolist())


def pin_bias_selects_only(orc):
    """The correction bias chooses experts but does not weight them.

    (a) a uniform shift of every bias keeps each token's selection, so the
        weights must not move; (b) a large bias on experts 0..k-1 forces them
        to be chosen for every token."""
    x, Wg, b, _, _ = small_layer(15, T=48, d=64, f=8, E=32, k=6, shared=False)
    r0 = orc.route(x, Wg, b, 6, 2.827, True)
    keep = r0.margin > 1e-4
    assert keep.sum() > 30
    r1 = orc.route(x, Wg, b + 0.25, 6, 2.827, True)
    assert np.array_equal(r0.ids[keep], r1.ids[keep])
    np.testing.assert_allclose(r0.weights[keep], r1.weights[keep], rtol=1e-12)
    bb = b.copy()
    bb[:6] += 10.0
    r2 = orc.route(x, Wg, bb, 6, 2.827, True)
    assert all(sorted(row) == list(range(6)) for row in r2.ids.tolist())


def pin_k_equals_E(orc):
    """k = E: every expert is chosen; with zero bias the slot order is the score
    order, so the weights are non-increasing along the slots."""
    x, Wg, _, _, _ = small_layer(16, T=10, d=32, f=8, E=8, k=8, shared=False)
    r = orc.route(x, Wg, np.zeros(8), 8, 2.827, True)
    assert all(sorted(row) == list(range(8)) for row in r.ids.tolist())
    assert np.all(np.diff(r.weights, axis=1) <= 0)
    np.testing.assert_allclose(r.weights.sum(axis=1), 2.827, rtol=1e-12)


def pin_identical_experts_closed_form(orc):
    """All routed experts equal to one SwiGLU E: y = 2.827 * E(x) with a zero
    shared expert, and 3.827 * E(x) when the shared expert is E too, for any
    routing."""
    T, d, f, E, k = 7, 32, 12, 9, 3
    x, Wg, b, ex, _ = small_layer(17, T, d, f, E, k, shared=False)
    one = ex[0]
    same = [one] * E
    ge, _ = _getters(same, None)
    e_x = orc.swiglu_expert(x, *one)
    zero = tuple(np.zeros_like(m) for m in one)
    y0, _ = orc.forward(x, Wg, b, ge, lambda: {"gate": zero[0], "up": zero[1], "down": zero[2]},
                        k, 2.827, True, "bf16", 1)
    np.testing.assert_allclose(y0, 2.827 * e_x, rtol=1e-10, atol=1e-12)
    y1, _ = orc.forward(x, Wg, b, ge, lambda: {"gate": one[0], "up": one[1], "down": one[2]},
                        k, 2.827, True, "bf16", 1)
    np.testing.assert_allclose(y1, 3.827 * e_x, rtol=1e-10, atol=1e-12)


def pin_textbook_values(orc):
    """sigmoid and silu at points with known values."""
    s = orc.sigmoid(np.array([0.0, 1.0, -1.0, 40.0, -800.0]))
    np.testing.assert_allclose(s, [0.5, 0.7310585786300049, 0.2689414213699951, 1.0, 0.0],
                               rtol=1e-15, atol=1e-300)
    z = orc.silu(np.array([0.0, 1.0, -1.0, 2.0, -800.0]))
    np.testing.assert_allclose(z, [0.0, 0.7310585786300049, -0.2689414213699951,
                                   1.7615941559557649, 0.0], rtol=1e-15, atol=1e-300)


def pin_printed_counts(orc):
    """Parameter counts and per-rank weight sizes the pages print."""
    g = json.load(open(os.path.join(GOLDEN, "printed_counts.json")))
    cfg = json.load(open(os.path.join(GOLDEN, "k2_config.json")))
    d, f, E = cfg["hidden_size"], cfg["moe_intermediate_size"], cfg["n_routed_experts"]
    per = orc.down_proj_params(d, f)
    assert per == g["down_proj_params_per_expert"]["value"]
    assert per * E == g["down_proj_params_per_layer"]["value"]
    assert per * E * g["moe_blocks"]["value"] == g["down_proj_params_model"]["value"]
    assert cfg["num_hidden_layers"] - cfg["first_k_dense_replace"] == g["moe_blocks"]["value"]
    for key in ("mlp_gb_per_rank_ep128_dsv3", "mlp_gb_per_rank_ep128_k2"):
        it = g[key]
        n = it["routed_per_rank"] + it["shared_per_rank"]
        gb = n * it["moe_layers"] * orc.expert_params(d, f) * 1 / 1e9  # FP8: 1 byte/param
        assert abs(gb - it["value"]) / it["value"] < 0.08, (key, gb)


def pin_act_quant(orc):
    """Dynamic activation quantisation: the largest |v| of each 128-group maps
    to +-448, and every element is within half an e4m3 step of its value."""
    r = _rng(18)
    v = (r.standard_normal((9, 384)) * np.array([1e-3, 1.0, 300.0])[r.integers(0, 3, (9, 1))]).astype(np.float32)
    v[3, 128:256] = 0.0
    codes, s = orc.act_quant(v)
    for i in range(v.shape[0]):
        for g in range(3):
            grp = v[i, g * 128:(g + 1) * 128]
            if np.all(grp == 0):
                assert s[i, g] == 1.0 and np.all(codes[i, g * 128:(g + 1) * 128] & 0x7F == 0)
                continue
            j = int(np.argmax(np.abs(grp)))
            assert codes[i, g * 128 + j] & 0x7F == 0x7E
    deq = orc.act_dequant(codes, s)
    sc = np.repeat(s.astype(np.float64), 128, axis=1)
    bound = np.maximum(np.abs(v) * 2.0 ** -4, sc * 2.0 ** -10)
    assert np.all(np.abs(deq - v) <= bound * (1 + 1e-6))


def pin_fp8_exact_grid(orc):
    """Values already on the e4m3 grid with power-of-two scales quantise
    losslessly: weight dequant is exact and activation quant round-trips."""
    r = _rng(19)
    codes = r.integers(0, 0x7E, size=(256, 128), dtype=np.int64).astype(np.uint8)
    codes[0, 0] = 0x7E  # each group of a row gets a 448 so amax/448 is the scale
    scales = 2.0 ** r.integers(-12, -4, size=(2, 1)).astype(np.float64)
    w = orc.weight_dequant(codes, scales.astype(np.float32))
    exp = e4.decode(codes) * np.repeat(np.repeat(scales, 128, 0), 128, 1)
    assert np.array_equal(w, exp)
    rows = e4.decode(codes[:4]).astype(np.float64)
    rows[:, 0] = 448.0
    rows *= 2.0 ** -7
    c2, s2 = orc.act_quant(rows.astype(np.float32))
    assert np.all(s2 == np.float32(2.0 ** -7))
    assert np.array_equal(orc.act_dequant(c2, s2), rows)


# ------------------------------------------------------ group-limited routing
def pin_group_route_vs_brute(orc):
    """Group-limited routing (n_group > 1) equals the scalar-loop router, for
    groups of several experts and of one expert each."""
    for E, ng, tg, k in ((24, 6, 2, 4), (16, 4, 3, 5), (12, 12, 5, 3), (32, 8, 4, 8)):
        x, Wg, b, _, _ = small_layer(21 + E, T=6, d=32, f=8, E=E, k=k, shared=False)
        b = b * 10.0  # a wider bias spread: group choices that differ from the plain top-k
        r = orc.route(x, Wg, b, k, 2.827, True, ng, tg)
        for t in range(x.shape[0]):
            ids, w = brute.route_token(x[t], Wg, b, k, 2.827, True, ng, tg)
            assert list(r.ids[t]) == ids, (E, ng, tg, t, r.ids[t], ids)
            np.testing.assert_allclose(r.weights[t], w, rtol=1e-12, atol=0)


def pin_group_identities(orc):
    """One group, or every group kept, is the plain top-k: the same ids and
    weights as a full sort of the keys (ties to the lower index)."""
    x, Wg, b, _, _ = small_layer(31, T=40, d=24, f=8, E=16, k=4, shared=False)
    keys = (_sig32(x @ Wg.T) + b.astype(np.float32)).astype(np.float32)
    plain = np.argsort(-keys.astype(np.float64), axis=1, kind="stable")[:, :4]
    for ng, tg in ((1, 1), (4, 4), (16, 16)):
        r = orc.route(x, Wg, b, 4, 2.827, True, ng, tg)
        assert np.array_equal(r.ids, plain), (ng, tg)
        assert np.all(np.isinf(r.group_margin))


def _sig32(l):
    l32 = np.asarray(l, np.float64).astype(np.float32).astype(np.float64)
    return (1.0 / (1.0 + np.exp(-l32))).astype(np.float32)


def pin_group_forced(orc):
    """A +10 bias on every expert of groups 1 and 4 (of 6) with topk_group = 2:
    those two groups are kept for every token, all chosen experts come from
    them, their weights are the bias-free normalised scores, and the group
    margin is about 10."""
    E, ng, k = 24, 6, 4
    x, Wg, b, _, _ = small_layer(41, T=30, d=32, f=8, E=E, k=k, shared=False)
    b = b.copy()
    forced = np.r_[4:8, 16:20]
    b[forced] += 10.0
    r = orc.route(x, Wg, b, k, 2.827, True, ng, 2)
    assert np.all(np.isin(r.ids, forced))
    sc = 1.0 / (1.0 + np.exp(-(x @ Wg.T)))
    sel = np.take_along_axis(sc, r.ids, axis=1)
    np.testing.assert_allclose(r.weights, 2.827 * sel / sel.sum(1, keepdims=True), rtol=1e-12)
    assert np.all(r.group_margin > 9.0)


def pin_group_invariants(orc):
    """On many tokens: the chosen experts span at most topk_group groups;
    every kept group's score (its two largest keys, added in float32) is at
    least every dropped group's; and the chosen ids are the top-k of the keys
    of the kept groups' experts."""
    E, ng, tg, k = 32, 8, 3, 6
    gs = E // ng
    x, Wg, b, _, _ = small_layer(51, T=200, d=16, f=8, E=E, k=k, shared=False)
    b = b * 10.0
    r = orc.route(x, Wg, b, k, 2.827, True, ng, tg)
    keys = r.keys.astype(np.float32)
    for t in range(x.shape[0]):
        g_of = r.ids[t] // gs
        assert len(set(g_of.tolist())) <= tg
        top2 = []
        for g in range(ng):
            kk = sorted(keys[t, g * gs:(g + 1) * gs].tolist(), reverse=True)
            top2.append(float(np.float32(kk[0]) + np.float32(kk[1])))
        kept = sorted(range(ng), key=lambda g: (-top2[g], g))[:tg]
        assert set(g_of.tolist()) <= set(kept)
        assert min(top2[g] for g in kept) >= max(top2[g] for g in range(ng) if g not in kept)
        cand = [e for e in range(E) if e // gs in kept]
        want = sorted(cand, key=lambda e: (-float(keys[t, e]), e))[:k]
        assert list(r.ids[t]) == want


def pin_group_tie_rule(orc):
    """Equal group scores keep the lower group: with a zero router every score
    is 1/2, so the keys are 1/2 + bias; groups 1 and 3 (of 4) get the same two
    largest biases, and topk_group = 1 must keep group 1."""
    E, ng, d = 16, 4, 8
    x = np.ones((3, d))
    Wg = np.zeros((E, d))
    b = np.zeros(E)
    b[[5, 6]] = [0.25, 0.125]     # group 1
    b[[13, 15]] = [0.125, 0.25]   # group 3: the same two values
    b[[0, 8]] = [0.2, 0.2]        # groups 0 and 2: lower sums
    r = orc.route(x, Wg, b, 2, 2.827, True, ng, 1)
    assert np.all(r.ids == np.array([5, 6]))
    assert np.all(r.group_margin == 0.0)


ALL_PINS = [pin_route_vs_brute, pin_layer_vs_brute_bf16, pin_layer_vs_brute_fp8,
            pin_weights_sum, pin_bias_selects_only, pin_k_equals_E,
            pin_identical_experts_closed_form, pin_textbook_values, pin_printed_counts,
            pin_act_quant, pin_fp8_exact_grid, pin_dense_ffn_vs_brute,
            pin_group_route_vs_brute, pin_group_identities, pin_group_forced,
            pin_group_invariants, pin_group_tie_rule]
