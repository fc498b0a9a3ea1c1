"""Float64 numpy oracle of the Kimi K2 routed-MoE layer forward pass.

Test infrastructure only (see the package docstring): the product path never
imports this module.

What the layer computes, and where the pages fix it:
  * router over n_routed_experts = 384 experts of hidden_size = 7168 inputs,
    scoring_func = sigmoid, topk_method = noaux_tc, n_group = topk_group = 1,
    num_experts_per_tok = 8, norm_topk_prob = true,
    routed_scaling_factor = 2.827, n_shared_experts = 1,
    moe_intermediate_size = 2048 -- "Kimi K2 Base" model card (raw config
    field table) and "Kimi K2 0905" model card (raw config fields).
  * each expert is the SwiGLU MLP down_proj(act_fn(gate_proj(x)) * up_proj(x))
    with act_fn = silu (hidden_act), no biases, weights held [out, in]
    -- "Kimi K2 · Down projection" (OpenModelAtlas): the module formula, the
    "no bias parameter" note and the [out, in] layout note.
  * FP8 variant: e4m3 weights with one scale per 128x128 block, dynamic
    activation scheme -- the same page's config.json quantization_config
    excerpt and its "one scale per 128 x 128 block" evidence note.

Readings taken where the pages are silent (the library follows the same ones):
  R1 router weight fp32, logits accumulated exactly (float64 here).
  R2 noaux_tc: key = sigmoid score + e_score_correction_bias; the bias only
     chooses experts, the weights use the unbiased scores.
  R3 top-k order: key descending, equal keys -> lower expert index first.
  R4 selection is decided on float32 keys (the precision the kernel decides
     in): logit rounded to fp32, sigmoid of it rounded to fp32, fp32 add of
     the fp32 bias.
  R5 normalise over the k selected unbiased scores, then multiply by 2.827.
  R6 shared expert: intermediate moe_intermediate_size * n_shared_experts,
     weight 1, not scaled by 2.827.
  R7 FP8: W = decode(q) * s_block; activations quantised per token per 128
     columns: s = amax/448 (fp32 divide), q = e4m3(v/s) (fp32 divide,
     nearest-even, saturating), amax = 0 -> s = 1; x is quantised before
     gate/up, the fp32 h = silu(g)*u before down. The router stays fp32 on
     the BF16 x.
  R19 group-limited routing (n_group > 1): contiguous groups of E / n_group
     experts, group score = float32 sum of the group's two largest keys, the
     topk_group best groups kept (ties to the lower group), top-k over their
     experts only (group_filter). K2 itself has n_group = 1.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, Optional, Sequence

import numpy as np

from . import e4m3

GROUP = 128  # FP8 block edge (weight_block_size [128, 128])


# --------------------------------------------------------------------------
# Router
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, router_weight: np.ndarray) -> np.ndarray:
    """logits[t, e] = sum_i x[t, i] * W_g[e, i], accumulated in float64 (R1)."""
    return np.asarray(x, np.float64) @ np.asarray(router_weight, np.float64).T


def sigmoid(z: np.ndarray) -> np.ndarray:
    """scoring_func = sigmoid: 1 / (1 + exp(-z)) in float64."""
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def selection_keys(logits: np.ndarray, bias: np.ndarray) -> np.ndarray:
    """float32 selection key = fp32(sigmoid(fp32(logit))) + fp32(bias)  (R2, R4)."""
    l32 = np.asarray(logits, np.float64).astype(np.float32)
    s32 = sigmoid(l32.astype(np.float64)).astype(np.float32)
    return s32 + np.asarray(bias, np.float32)[None, :]


def topk_by_key(key: np.ndarray, k: int):
    """Indices of the k largest keys per row, key descending, ties to the lower
    index (R3); margin = k-th key minus (k+1)-th key (inf when k == E)."""
    key = np.asarray(key)
    order = np.argsort(-key, axis=1, kind="stable")
    ids = order[:, :k]
    ks = np.take_along_axis(key, order, axis=1).astype(np.float64)
    if k < key.shape[1]:
        margin = ks[:, k - 1] - ks[:, k]
    else:
        margin = np.full(key.shape[0], np.inf)
    return ids.astype(np.int64), margin


def group_filter(keys: np.ndarray, n_group: int, topk_group: int):
    """Group-limited routing (config fields n_group, topk_group: "Kimi K2
    Base" raw config table, both 1 for K2; why grouping exists and why K2
    drops it: "Behind Kimi-K2's Config" §2.4). The pages give no group rule;
    this library's reading (R19):
      * the E experts form n_group contiguous groups of E / n_group;
      * a group's score is the float32 sum of its two largest selection keys
        (its one key for groups of one expert), decided in float32 as the
        keys are (R4);
      * the topk_group groups with the largest scores are kept, ties to the
        lower group index; every expert of the other groups drops out of the
        top-k (its key becomes -inf).
    With n_group = 1 the one group is kept and nothing changes.
    Returns (keys with the dropped experts at -inf, group margin [T] = the
    topk_group-th minus the next group score, inf when every group is kept).
    """
    keys = np.asarray(keys, np.float32)
    T, E = keys.shape
    if n_group < 1 or E % n_group or not 1 <= topk_group <= n_group:
        raise ValueError("n_group must divide E and 1 <= topk_group <= n_group")
    gs = E // n_group
    by_group = -np.sort(-keys.reshape(T, n_group, gs), axis=2)  # each group's keys, descending
    if gs >= 2:
        gscore = (by_group[:, :, 0] + by_group[:, :, 1]).astype(np.float32)  # float32 add
    else:
        gscore = by_group[:, :, 0]
    order = np.argsort(-gscore.astype(np.float64), axis=1, kind="stable")  # ties: lower group
    kept = np.zeros((T, n_group), bool)
    np.put_along_axis(kept, order[:, :topk_group], True, axis=1)
    masked = np.where(np.repeat(kept, gs, axis=1), keys, np.float32(-np.inf)).astype(np.float32)
    if topk_group < n_group:
        gs_sorted = np.take_along_axis(gscore.astype(np.float64), order, axis=1)
        gmargin = gs_sorted[:, topk_group - 1] - gs_sorted[:, topk_group]
    else:
        gmargin = np.full(T, np.inf)
    return masked, gmargin


@dataclasses.dataclass
class Routing:
    ids: np.ndarray       # [T, k] int64, slot order = key descending
    weights: np.ndarray   # [T, k] float64, sum = routed_scaling_factor (norm on)
    scores: np.ndarray    # [T, E] float64 unbiased sigmoid scores
    keys: np.ndarray      # [T, E] float32 selection keys (before the group filter)
    margin: np.ndarray    # [T] float64, k-th minus (k+1)-th key among the kept experts
    group_margin: Optional[np.ndarray] = None  # [T] topk_group-th minus next group score


def route(x, router_weight, bias, k: int, routed_scaling_factor: float = 2.827,
          norm_topk_prob: bool = True, n_group: int = 1, topk_group: int = 1) -> Routing:
    """Router of the layer: sigmoid scores, noaux_tc biased top-k (after the
    group filter, which keeps every expert when n_group = 1), normalise,
    scale."""
    logits = router_logits(x, router_weight)
    scores = sigmoid(logits)
    keys = selection_keys(logits, bias)
    masked, gmargin = group_filter(keys, n_group, topk_group)
    ids, margin = topk_by_key(masked, k)
    w = routing_weights(scores, ids, routed_scaling_factor, norm_topk_prob)
    return Routing(ids=ids, weights=w, scores=scores, keys=keys, margin=margin,
                   group_margin=gmargin)


def routing_weights(scores: np.ndarray, ids: np.ndarray, routed_scaling_factor: float = 2.827,
                    norm_topk_prob: bool = True) -> np.ndarray:
    """Weights of the chosen experts ids [T, k] from the unbiased scores [T, E]
    (R2: the bias never enters): normalised over the k chosen scores when
    norm_topk_prob ("Kimi K2 Base" raw config: norm_topk_prob true), then
    times routed_scaling_factor (2.827), R5."""
    sel = np.take_along_axis(np.asarray(scores, np.float64), np.asarray(ids, np.int64), axis=1)
    if norm_topk_prob:
        w = sel / sel.sum(axis=1, keepdims=True)
    else:
        w = sel.copy()
    return w * routed_scaling_factor


# --------------------------------------------------------------------------
# Experts
# --------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """hidden_act = silu: z * sigmoid(z) = z / (1 + exp(-z))."""
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_expert(xr: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
                  w_down: np.ndarray) -> np.ndarray:
    """down_proj(silu(gate_proj(x)) * up_proj(x)) for rows xr [n, d].

    Weights are [out, in]: gate/up [f, d], down [d, f]; no biases.
    """
    xr = np.asarray(xr, np.float64)
    g = xr @ np.asarray(w_gate, np.float64).T
    u = xr @ np.asarray(w_up, np.float64).T
    h = silu(g) * u
    return h @ np.asarray(w_down, np.float64).T


def act_quant(v: np.ndarray, group: int = GROUP):
    """Dynamic per-row, per-128-column e4m3 quantisation (R7).

    v is float32 [n, c]. Returns (codes uint8 [n, c], scales float32 [n, c/128]).
    Every decision is made in float32: amax, s = amax / 448, v / s.
    """
    v = np.asarray(v, np.float32)
    n, c = v.shape
    vg = v.reshape(n, c // group, group)
    amax = np.abs(vg).max(axis=2)
    s = (amax / np.float32(448.0)).astype(np.float32)
    s = np.where(amax == 0, np.float32(1.0), s).astype(np.float32)
    q = (vg / s[:, :, None]).astype(np.float32)
    codes = e4m3.encode(q.astype(np.float64)).reshape(n, c)
    return codes, s


def act_dequant(codes: np.ndarray, scales: np.ndarray, group: int = GROUP) -> np.ndarray:
    n, c = codes.shape
    return (e4m3.decode(codes).reshape(n, c // group, group)
            * np.asarray(scales, np.float64)[:, :, None]).reshape(n, c)


def weight_dequant(codes: np.ndarray, scales: np.ndarray, block: int = GROUP) -> np.ndarray:
    """W[r, c] = decode(q[r, c]) * s[r // 128, c // 128] in float64."""
    r, c = codes.shape
    w = e4m3.decode(codes).reshape(r // block, block, c // block, block)
    return (w * np.asarray(scales, np.float64)[:, None, :, None]).reshape(r, c)


def swiglu_expert_fp8(xr: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
                      w_down: np.ndarray) -> np.ndarray:
    """FP8 expert: dequantised weights (given), activations quantised before
    gate/up (x) and before down (the fp32-rounded h), R7."""
    xq, xs = act_quant(np.asarray(xr, np.float32))
    xd = act_dequant(xq, xs)
    g = xd @ np.asarray(w_gate, np.float64).T
    u = xd @ np.asarray(w_up, np.float64).T
    h = silu(g) * u
    hq, hs = act_quant(h.astype(np.float32))
    hd = act_dequant(hq, hs)
    return hd @ np.asarray(w_down, np.float64).T


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------
ExpertFn = Callable[[int], Dict[str, np.ndarray]]


def expert_matrices(mats: Dict[str, np.ndarray], fmt: str) -> Dict[str, np.ndarray]:
    """An expert's gate/up/down as float64 values: BF16 values widened, or FP8
    codes dequantised with their block scales (R7)."""
    if fmt == "bf16":
        return {n: np.asarray(mats[n], np.float64) for n in ("gate", "up", "down")}
    return {n: weight_dequant(mats[n], mats[n + "_scale"]) for n in ("gate", "up", "down")}


def expert_function(fmt: str):
    """The expert MLP of the weight format: swiglu_expert (BF16) or
    swiglu_expert_fp8 (activations quantised as R7 states)."""
    return swiglu_expert if fmt == "bf16" else swiglu_expert_fp8


def combine(pair_out: np.ndarray, weights: np.ndarray,
            shared_out: Optional[np.ndarray] = None) -> np.ndarray:
    """y[t] = sum_j w[t, j] * pair_out[t, j] + shared_out[t]: the routed
    outputs weighted and summed in slot order j = 0..k-1, then the shared
    expert at weight 1, not scaled (R6)."""
    pair_out = np.asarray(pair_out, np.float64)
    w = np.asarray(weights, np.float64)
    y = np.zeros((pair_out.shape[0], pair_out.shape[2]), np.float64)
    for j in range(pair_out.shape[1]):
        y += w[:, j:j + 1] * pair_out[:, j]
    if shared_out is not None:
        y += shared_out
    return y


def experts_combine(x: np.ndarray, ids: np.ndarray, weights: np.ndarray,
                    get_expert: ExpertFn, get_shared: Optional[Callable[[], Dict]],
                    fmt: str = "bf16", n_shared_experts: int = 1,
                    tokens: Optional[Sequence[int]] = None) -> np.ndarray:
    """y[t] = sum_j w[t, j] * E_{ids[t, j]}(x_t) + S(x_t) for the listed tokens.

    get_expert(e) returns routed expert e's matrices (BF16 values or FP8 codes
    plus scales), get_shared() the shared expert's ([f_s, d], [f_s, d],
    [d, f_s]). Pairs are evaluated expert by expert so each expert's weights
    are fetched once; every pair's output is the same expert formula, and the
    per-token sum runs in slot order j = 0..k-1, then the shared expert.
    """
    x = np.asarray(x, np.float64)
    toks = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens, np.int64)
    n, k = len(toks), ids.shape[1]
    ffn = expert_function(fmt)
    pair_out = np.zeros((n, k, x.shape[1]), np.float64)
    sub_ids = np.asarray(ids)[toks]
    for e in np.unique(sub_ids):
        rows, slots = np.nonzero(sub_ids == e)
        m = expert_matrices(get_expert(int(e)), fmt)
        pair_out[rows, slots] = ffn(x[toks[rows]], m["gate"], m["up"], m["down"])
    shared_out = None
    if get_shared is not None and n_shared_experts > 0:
        m = expert_matrices(get_shared(), fmt)
        shared_out = ffn(x[toks], m["gate"], m["up"], m["down"])
    return combine(pair_out, np.asarray(weights, np.float64)[toks], shared_out)


def dense_ffn(x: np.ndarray, mats: Dict[str, np.ndarray], fmt: str = "bf16") -> np.ndarray:
    """The model's dense FFN layer, its first layer ("Behind Kimi-K2's Config"
    §2.3: first_k_dense = 1; "Kimi K2 Base" raw config fields:
    first_k_dense_replace 1, intermediate_size 18432, hidden_act silu):
    y = down(silu(gate x) * up x) over intermediate_size columns, no router.
    The pages print this formula for the experts ("Kimi K2 · Down
    projection"); the dense layer is read as the same MLP. mats holds
    gate [i, d], up [i, d], down [d, i] (BF16 values, or FP8 codes with their
    *_scale block scales, dequantised and with x and h quantised as for the
    experts)."""
    x = np.asarray(x, np.float64)
    m = expert_matrices(mats, fmt)
    return expert_function(fmt)(x, m["gate"], m["up"], m["down"])


def forward(x, router_weight, bias, get_expert: ExpertFn, get_shared, k: int,
            routed_scaling_factor: float = 2.827, norm_topk_prob: bool = True,
            fmt: str = "bf16", n_shared_experts: int = 1,
            tokens: Optional[Sequence[int]] = None, n_group: int = 1, topk_group: int = 1):
    """Full layer: route every token, then evaluate the listed tokens (all by
    default). Returns (y float64 [n, d], Routing over all T tokens)."""
    r = route(x, router_weight, bias, k, routed_scaling_factor, norm_topk_prob, n_group,
              topk_group)
    y = experts_combine(x, r.ids, r.weights, get_expert, get_shared, fmt,
                        n_shared_experts, tokens)
    return y, r


# --------------------------------------------------------------------------
# Sizes printed on the pages
# --------------------------------------------------------------------------
def down_proj_params(hidden_size: int, moe_intermediate_size: int) -> int:
    """Parameters of one expert's down projection: a [hidden, intermediate]
    matrix with no bias."""
    return hidden_size * moe_intermediate_size


def expert_params(hidden_size: int, moe_intermediate_size: int) -> int:
    """gate_proj + up_proj + down_proj of one SwiGLU expert."""
    return 3 * hidden_size * moe_intermediate_size
