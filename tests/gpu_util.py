"""Helpers shared by the GPU parity tests: build a layer on the device from
the seeded generator, run it through the C ABI, and compare with the oracle
on the host (the oracle gets host copies of the same generated tensors)."""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

import synth
from oracle import moe as orc

NEAR_TIE = 1e-5  # k-th vs (k+1)-th key gap below which either choice is correct
TOL = {"bf16": 1e-2, "fp8": 3e-2}


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


@dataclasses.dataclass
class Layer:
    shape: synth.LayerShape
    fmt: str
    x: torch.Tensor
    Wg: torch.Tensor
    b: torch.Tensor
    ew: synth.ExpertWeights


def make_layer(shape, T, fmt="bf16", seed=synth.SEED, device="cuda", identical=False,
               shared_zero=False, router_row_scale=None, bias_std=0.01) -> Layer:
    x = synth.make_tokens(shape, T, seed, device)
    Wg, b = synth.make_router(shape, seed, device, bias_std, router_row_scale)
    ew = synth.make_experts(shape, seed, device, fmt, identical, shared_zero)
    return Layer(shape, fmt, x, Wg, b, ew)


def create_handle(smoe, layer: Layer, max_tokens: int, device: int = 0):
    s = layer.shape
    cfg = smoe.moe_config_init_k2(
        hidden_size=s.hidden_size, moe_intermediate_size=s.moe_intermediate_size,
        n_routed_experts=s.n_routed_experts, num_experts_per_tok=s.num_experts_per_tok,
        n_shared_experts=s.n_shared_experts, routed_scaling_factor=s.routed_scaling_factor,
        norm_topk_prob=int(s.norm_topk_prob), max_tokens=max_tokens,
        weight_format=smoe.MOE_WEIGHT_BF16 if layer.fmt == "bf16" else smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    h = smoe.moe_create(cfg, device)
    ew = layer.ew
    smoe.moe_load_weights(h, layer.Wg, layer.b, ew.gate, ew.up, ew.down, ew.shared_gate,
                          ew.shared_up, ew.shared_down, ew.gate_scale, ew.up_scale, ew.down_scale,
                          ew.shared_gate_scale, ew.shared_up_scale, ew.shared_down_scale)
    torch.cuda.synchronize()
    return h


def run(smoe, h, layer: Layer, x: Optional[torch.Tensor] = None, forced=None):
    x = layer.x if x is None else x
    T, k = x.shape[0], layer.shape.num_experts_per_tok
    y = torch.empty_like(x)
    ids = torch.full((T, k), -1, dtype=torch.int32, device=x.device)
    w = torch.zeros((T, k), dtype=torch.float32, device=x.device)
    smoe.moe_forward(h, x, y, topk_ids_out=ids, topk_weights_out=w, forced_topk_ids=forced,
                     flags=smoe.MOE_FLAG_SYNC_CHECK)
    return y, ids, w


def _getters(layer: Layer):
    cache = {}

    def ge(e):
        if e not in cache:
            m = synth.expert_slice(layer.ew, e)
            cache[e] = {n: (to_np(v) if v.dtype != torch.uint8 else v.numpy()) for n, v in m.items()}
        return cache[e]

    def gs():
        m = synth.shared_slice(layer.ew)
        return {n: (to_np(v) if v.dtype != torch.uint8 else v.numpy()) for n, v in m.items()}

    return ge, (gs if layer.shape.n_shared_experts > 0 else None)


def oracle_route(layer: Layer, x: Optional[torch.Tensor] = None):
    s = layer.shape
    xx = to_np(layer.x if x is None else x).astype(np.float64)
    return orc.route(xx, to_np(layer.Wg).astype(np.float64), to_np(layer.b).astype(np.float64),
                     s.num_experts_per_tok, s.routed_scaling_factor, s.norm_topk_prob)


def oracle_outputs(layer: Layer, ids: np.ndarray, weights: np.ndarray, tokens: Sequence[int],
                   x: Optional[torch.Tensor] = None) -> np.ndarray:
    s = layer.shape
    xx = to_np(layer.x if x is None else x).astype(np.float64)
    ge, gs = _getters(layer)
    return orc.experts_combine(xx, ids, weights, ge, gs, layer.fmt, s.n_shared_experts, tokens)


@dataclasses.dataclass
class Report:
    near_ties: int
    id_mismatch_outside_ties: int
    invalid_tie_choices: int
    weight_max_rel: float
    y_rel_err: float
    compared_tokens: int
    order_swaps: int = 0


def compare(layer: Layer, y_gpu, ids_gpu, w_gpu, tokens: Optional[Sequence[int]] = None,
            x=None) -> Report:
    """Routing for every token; outputs for `tokens` (all by default).

    What is unique is compared exactly: the SET of chosen experts of every
    token whose k-th and (k+1)-th oracle keys differ by at least NEAR_TIE.
    What is not unique is checked for validity: a near-tie token may choose
    another expert at the boundary, but every chosen expert's oracle key must
    be within NEAR_TIE of the oracle's k-th key; and the slot order (key
    descending) may swap experts whose keys are within NEAR_TIE, so the
    oracle keys along the GPU's slots must be non-increasing within NEAR_TIE.
    Weights are compared per expert id; outputs for tokens whose set matches.
    """
    r = oracle_route(layer, x)
    T = r.ids.shape[0]
    k = layer.shape.num_experts_per_tok
    gid = to_np(ids_gpu).astype(np.int64)
    gw = to_np(w_gpu).astype(np.float64)
    tie = r.margin < NEAR_TIE
    same_set = np.array([set(gid[t]) == set(r.ids[t]) for t in range(T)])
    mism = int(np.sum(~same_set & ~tie))
    invalid = 0
    swaps = 0
    for t in range(T):
        kt = r.keys[t].astype(np.float64)
        along = kt[gid[t]]
        if np.any(np.diff(along) > NEAR_TIE) or len(set(gid[t])) != k:
            invalid += 1
        if not np.array_equal(gid[t], r.ids[t]) and same_set[t]:
            swaps += 1
        if not same_set[t] and tie[t]:
            kth = np.sort(kt)[::-1][k - 1]
            if np.any(along < kth - NEAR_TIE):
                invalid += 1
    ok = same_set
    wrel = 0.0
    for t in np.nonzero(ok)[0]:
        og = dict(zip(r.ids[t].tolist(), r.weights[t].tolist()))
        for e, wv in zip(gid[t].tolist(), gw[t].tolist()):
            wrel = max(wrel, abs(wv - og[e]) / abs(og[e]))
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    toks = toks[ok[toks]]
    yo = oracle_outputs(layer, r.ids, r.weights, toks, x)
    yg = to_np(y_gpu).astype(np.float64)[toks]
    err = float(np.max(np.abs(yg - yo)) / max(np.max(np.abs(yo)), 1e-30)) if len(toks) else 0.0
    return Report(int(tie.sum()), mism, invalid, wrel, err, len(toks), swaps)
