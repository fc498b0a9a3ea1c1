"""Helpers shared by the GPU parity tests: build a layer on the device from
the seeded generator, run it through the C ABI, and compare with the oracle
on the host (the oracle gets host copies of the same generated tensors).

Comparison rules (the acceptance rule of the workload spec):
  * routing of every token: the SET of chosen experts equals the oracle's,
    except near-ties (k-th and (k+1)-th oracle keys within NEAR_TIE), which
    may choose either side but must stay a valid top-k within NEAR_TIE; slots
    in key order within NEAR_TIE; weights to 1e-5 relative;
  * outputs on a seeded sample (every token up to 512, else 512 of them,
    always the first and the last) plus every near-tie token, all evaluated
    by the oracle under the experts the GPU chose and the oracle's weights
    for them (for a token whose set equals the oracle's this is the oracle's
    own output);
  * max|gpu - oracle| / max|oracle| <= TOL[fmt].
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Dict, Iterable, Optional, Sequence

import numpy as np
import torch

import synth
from oracle import moe as orc

NEAR_TIE = 1e-5  # k-th vs (k+1)-th key gap below which either choice is correct
TOL = {"bf16": 1e-2, "fp8": 3e-2}
N_SAMPLE = 512


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 (or uint8 codes) host copy of a tensor."""
    t = t.detach().cpu()
    if t.dtype == torch.uint8:
        return t.numpy()
    return t.to(torch.float64).numpy()


def sample_tokens(T: int, n: int = N_SAMPLE, seed: int = 0x5EED) -> np.ndarray:
    """Every token when T <= n; else the first and last token and n - 2 others
    from a fixed permutation (so the samples of different T overlap)."""
    if T <= n:
        return np.arange(T)
    perm = np.random.default_rng(seed).permutation(max(T, 1 << 16))
    pick = perm[(perm > 0) & (perm < T - 1)][: n - 2]
    return np.unique(np.concatenate([[0, T - 1], pick]))


@dataclasses.dataclass
class Layer:
    shape: synth.LayerShape
    fmt: str
    x: torch.Tensor
    Wg: torch.Tensor
    b: torch.Tensor
    ew: synth.ExpertWeights
    cache: Optional["OracleCache"] = None


def make_layer(shape, T, fmt="bf16", seed=synth.SEED, device="cuda", identical=False,
               shared_zero=False, router_row_scale=None, bias_std=0.01) -> Layer:
    x = synth.make_tokens(shape, T, seed, device)
    Wg, b = synth.make_router(shape, seed, device, bias_std, router_row_scale)
    ew = synth.make_experts(shape, seed, device, fmt, identical, shared_zero)
    return Layer(shape, fmt, x, Wg, b, ew)


def create_handle(smoe, layer: Layer, max_tokens: int, device: int = 0,
                  single_launch_max_tokens: int = 0):
    s = layer.shape
    cfg = smoe.moe_config_init_k2(
        hidden_size=s.hidden_size, moe_intermediate_size=s.moe_intermediate_size,
        n_routed_experts=s.n_routed_experts, num_experts_per_tok=s.num_experts_per_tok,
        n_shared_experts=s.n_shared_experts, routed_scaling_factor=s.routed_scaling_factor,
        norm_topk_prob=int(s.norm_topk_prob), max_tokens=max_tokens,
        n_group=s.n_group, topk_group=s.topk_group,
        single_launch_max_tokens=single_launch_max_tokens,
        weight_format=smoe.MOE_WEIGHT_BF16 if layer.fmt == "bf16" else smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    h = smoe.moe_create(cfg, device)
    ew = layer.ew
    smoe.moe_load_weights(h, layer.Wg, layer.b, ew.gate, ew.up, ew.down, ew.shared_gate,
                          ew.shared_up, ew.shared_down, ew.gate_scale, ew.up_scale, ew.down_scale,
                          ew.shared_gate_scale, ew.shared_up_scale, ew.shared_down_scale)
    torch.cuda.synchronize()
    return h


@dataclasses.dataclass
class Run:
    y: torch.Tensor
    ids: torch.Tensor
    w: torch.Tensor
    offsets: Optional[torch.Tensor] = None
    pair_rows: Optional[torch.Tensor] = None

    def __iter__(self):  # y, ids, w = run(...)
        return iter((self.y, self.ids, self.w))

    def __getitem__(self, i):  # run(...)[0] is y
        return (self.y, self.ids, self.w)[i]


def run(smoe, h, layer: Layer, x: Optional[torch.Tensor] = None, forced=None,
        permutation: bool = False, flags: int = 0) -> Run:
    x = layer.x if x is None else x
    T, k, E = x.shape[0], layer.shape.num_experts_per_tok, layer.shape.n_routed_experts
    y = torch.empty_like(x)
    ids = torch.full((T, k), -1, dtype=torch.int32, device=x.device)
    w = torch.zeros((T, k), dtype=torch.float32, device=x.device)
    off = pr = None
    if permutation:
        off = torch.full((E + 1,), -1, dtype=torch.int32, device=x.device)
        pr = torch.full((T, k), -1, dtype=torch.int32, device=x.device)
    smoe.moe_forward(h, x, y, topk_ids_out=ids, topk_weights_out=w, forced_topk_ids=forced,
                     flags=smoe.MOE_FLAG_SYNC_CHECK | flags, expert_offsets_out=off,
                     pair_rows_out=pr)
    return Run(y, ids, w, off, pr)


# --------------------------------------------------------------- the oracle
def _expert_getter(layer: Layer):
    ew = layer.ew

    def get(e: int) -> Dict[str, np.ndarray]:
        m = synth.expert_slice(ew, e) if e >= 0 else synth.shared_slice(ew)
        return {n: f64(v) for n, v in m.items()}

    return get


def _workers() -> int:
    return max(1, min(8, (os.cpu_count() or 2) // 2))


class OracleCache:
    """The oracle evaluated for one layer, kept for reuse across the forwards
    of a test module: the routing of every token of layer.x, and each
    (token, expert) output E_e(x_t) and shared-expert output S(x_t) computed
    so far. A forward over T tokens uses layer.x[:T]; a token's routing and
    expert outputs do not depend on T. Missing outputs are computed expert
    by expert (each expert's matrices converted once per batch), experts in
    parallel threads."""

    def __init__(self, layer: Layer):
        self.layer = layer
        s = layer.shape
        self.x = f64(layer.x)
        self.E, self.k = s.n_routed_experts, s.num_experts_per_tok
        self.r = orc.route(self.x, f64(layer.Wg), f64(layer.b), s.num_experts_per_tok,
                           s.routed_scaling_factor, s.norm_topk_prob, s.n_group, s.topk_group)
        self.pair: Dict[tuple, np.ndarray] = {}
        self.shared: Dict[int, np.ndarray] = {}
        self._get = _expert_getter(layer)
        self._ffn = orc.expert_function(layer.fmt)

    def near_tie_candidates(self, t: int) -> np.ndarray:
        """Experts a near-tie token may validly choose: keys within NEAR_TIE of
        the k-th largest."""
        kt = self.r.keys[t].astype(np.float64)
        kth = np.sort(kt)[::-1][self.k - 1]
        return np.nonzero(kt >= kth - NEAR_TIE)[0]

    def prepare(self, tokens: Iterable[int], with_ties_below: Optional[int] = None):
        """Compute the outputs of the oracle's experts for `tokens`, and of
        every valid near-tie choice for the near-tie tokens below
        with_ties_below."""
        want = set()
        toks = np.asarray(sorted(set(int(t) for t in tokens)), np.int64)
        for t in toks:
            want.update((int(t), int(e)) for e in self.r.ids[t])
        if with_ties_below:
            for t in np.nonzero(self.r.margin[:with_ties_below] < NEAR_TIE)[0]:
                want.update((int(t), int(e)) for e in self.near_tie_candidates(t))
        shared_toks = set(toks.tolist()) | {t for t, _ in want}
        self._compute(want, shared_toks)

    def _compute(self, pairs, shared_toks):
        pairs = [p for p in pairs if p not in self.pair]
        shared_toks = sorted(t for t in shared_toks if t not in self.shared)
        by_e: Dict[int, list] = {}
        for t, e in pairs:
            by_e.setdefault(e, []).append(t)
        jobs = [(e, sorted(ts)) for e, ts in by_e.items()]
        if shared_toks and self.layer.shape.n_shared_experts > 0:
            jobs.append((-1, shared_toks))

        def work(job):
            e, ts = job
            m = orc.expert_matrices(self._get(e), self.layer.fmt)
            return e, ts, self._ffn(self.x[ts], m["gate"], m["up"], m["down"])

        with concurrent.futures.ThreadPoolExecutor(_workers()) as ex:
            for e, ts, out in ex.map(work, jobs):
                for i, t in enumerate(ts):
                    if e >= 0:
                        self.pair[(t, e)] = out[i]
                    else:
                        self.shared[t] = out[i]

    def outputs(self, tokens: Sequence[int], ids: np.ndarray, weights: np.ndarray) -> np.ndarray:
        """Oracle y for `tokens` under the given ids [T, k] and weights [T, k]."""
        toks = np.asarray(tokens, np.int64)
        need = {(int(t), int(e)) for t in toks for e in ids[t]}
        self._compute(need, set(toks.tolist()))
        pair_out = np.stack([np.stack([self.pair[(int(t), int(e))] for e in ids[t]])
                             for t in toks]) if len(toks) else np.zeros((0, ids.shape[1], 1))
        shared = None
        if self.layer.shape.n_shared_experts > 0:
            shared = np.stack([self.shared[int(t)] for t in toks])
        return orc.combine(pair_out, np.asarray(weights, np.float64)[toks], shared)


def cache_of(layer: Layer) -> OracleCache:
    if layer.cache is None:
        layer.cache = OracleCache(layer)
    return layer.cache


def oracle_route(layer: Layer, x: Optional[torch.Tensor] = None):
    """The oracle's routing of x (layer.x by default)."""
    s = layer.shape
    xx = f64(layer.x if x is None else x)
    return orc.route(xx, f64(layer.Wg), f64(layer.b), s.num_experts_per_tok,
                     s.routed_scaling_factor, s.norm_topk_prob, s.n_group, s.topk_group)


def oracle_outputs(layer: Layer, ids: np.ndarray, weights: np.ndarray, tokens: Sequence[int],
                   x: Optional[torch.Tensor] = None) -> np.ndarray:
    """Oracle outputs of `tokens` of layer.x[:T] under the given routing."""
    if x is not None:
        _check_prefix(layer, x)
    return cache_of(layer).outputs(tokens, np.asarray(ids), np.asarray(weights))


def _check_prefix(layer: Layer, x: torch.Tensor):
    T = x.shape[0]
    assert torch.equal(x, layer.x[:T]), "the oracle cache covers prefixes of layer.x only"


# ----------------------------------------------------------------- compare
@dataclasses.dataclass
class Report:
    T: int
    near_ties: int                 # tokens whose k-th and (k+1)-th oracle keys are within NEAR_TIE
    near_tie_other_choice: int     # near-tie tokens whose GPU set differs from the oracle's
    near_tie_compared: int         # near-tie tokens whose outputs were compared
    id_mismatch_outside_ties: int
    invalid_tie_choices: int
    weight_max_rel: float
    y_rel_err: float
    compared_tokens: int
    order_swaps: int = 0

    def line(self) -> str:
        return (f"T={self.T}: outputs compared on {self.compared_tokens} tokens, max rel err "
                f"{self.y_rel_err:.2e}; near-ties {self.near_ties} ({self.near_tie_other_choice} "
                f"chose the other side, {self.near_tie_compared} compared); weights max rel "
                f"{self.weight_max_rel:.1e}; id mismatches outside ties "
                f"{self.id_mismatch_outside_ties}, invalid tie choices {self.invalid_tie_choices}")


@dataclasses.dataclass
class RoutingCheck:
    tie: np.ndarray         # [T] near-tie tokens
    same_set: np.ndarray    # [T] GPU set == oracle set
    mismatch: int           # tokens outside the ties whose sets differ
    invalid: int            # tokens whose choice is not a valid top-k within NEAR_TIE
    swaps: int              # same set, other slot order
    ids_safe: np.ndarray    # GPU ids, or the oracle's where the GPU's are out of range
    w_ref: np.ndarray       # the oracle's weights for ids_safe
    weight_max_rel: float


def _group_scores(keys_t: np.ndarray, n_group: int) -> np.ndarray:
    """float32 sum of each contiguous group's two largest keys (one key for
    groups of one), as the group filter scores them."""
    g = -np.sort(-keys_t.astype(np.float32).reshape(n_group, -1), axis=1)
    return (g[:, 0] + g[:, 1]).astype(np.float32) if g.shape[1] >= 2 else g[:, 0]


def _valid_group_tie_choice(keys_t, ids_t, k, n_group, topk_group) -> bool:
    """A token whose kept groups are near-tied may keep another group: its
    experts must come from at most topk_group groups, each scoring within
    2 * NEAR_TIE of the oracle's topk_group-th group, and be the top-k of
    the keys of their own groups within NEAR_TIE."""
    E = keys_t.shape[0]
    gs = E // n_group
    gsc = _group_scores(keys_t, n_group).astype(np.float64)
    cut = np.sort(gsc)[::-1][topk_group - 1] - 2 * NEAR_TIE
    groups = np.unique(ids_t // gs)
    if len(groups) > topk_group or np.any(gsc[groups] < cut):
        return False
    members = np.concatenate([np.arange(g * gs, (g + 1) * gs) for g in groups])
    others = np.setdiff1d(members, ids_t)
    kk = keys_t.astype(np.float64)
    return not len(others) or kk[others].max() <= kk[ids_t].min() + NEAR_TIE


def check_routing(r, gid: np.ndarray, gw: np.ndarray, E: int, scale: float,
                  norm: bool, n_group: int = 1, topk_group: int = 1) -> RoutingCheck:
    """The GPU's ids [T, k] and weights against the oracle routing r (rows
    [0, T) of it): sets exact outside near-ties, near-tie choices valid,
    slots in key order within NEAR_TIE, weights against the oracle's weights
    for the same ids. With group-limited routing a token is also a near-tie
    when its topk_group-th and next group scores are within 2 * NEAR_TIE
    (a group score adds two keys)."""
    T, k = gid.shape
    keys, margin, oid = r.keys[:T], r.margin[:T], r.ids[:T]
    tie = margin < NEAR_TIE
    if n_group > 1 and r.group_margin is not None:
        tie = tie | (r.group_margin[:T] < 2 * NEAR_TIE)
    same_set = np.array([set(gid[t]) == set(oid[t]) for t in range(T)])
    mism = int(np.sum(~same_set & ~tie))
    invalid = swaps = 0
    for t in range(T):
        if len(set(gid[t])) != k or np.any(gid[t] < 0) or np.any(gid[t] >= E):
            invalid += 1
            continue
        kt = keys[t].astype(np.float64)
        along = kt[gid[t]]
        if np.any(np.diff(along) > NEAR_TIE):
            invalid += 1
            continue
        if not np.array_equal(gid[t], oid[t]) and same_set[t]:
            swaps += 1
        if not same_set[t] and tie[t]:
            if n_group > 1:
                if not _valid_group_tie_choice(keys[t], gid[t], k, n_group, topk_group):
                    invalid += 1
                continue
            kth = np.sort(kt)[::-1][k - 1]
            if np.any(along < kth - NEAR_TIE):
                invalid += 1
    # the oracle's weights for the experts the GPU chose (= the oracle's own
    # weights wherever the sets agree)
    valid = np.all((gid >= 0) & (gid < E), axis=1)
    ids_safe = np.where(valid[:, None], gid, oid)
    w_ref = orc.routing_weights(r.scores[:T], ids_safe, scale, norm)
    wrel = float(np.max(np.abs(gw - w_ref) / np.abs(w_ref))) if T else 0.0
    return RoutingCheck(tie, same_set, mism, invalid, swaps, ids_safe, w_ref, wrel)


def compare(layer: Layer, y_gpu, ids_gpu, w_gpu, tokens: Optional[Sequence[int]] = None,
            x=None) -> Report:
    """Routing of every token; outputs of `tokens` (default: sample_tokens(T))
    and of every near-tie token, under the GPU's ids (module docstring)."""
    gid = to_np(ids_gpu).astype(np.int64)
    T = gid.shape[0]
    if x is not None:
        _check_prefix(layer, x)
    c = cache_of(layer)
    s = layer.shape
    rc = check_routing(c.r, gid, to_np(w_gpu).astype(np.float64), c.E, s.routed_scaling_factor,
                       s.norm_topk_prob, s.n_group, s.topk_group)
    toks = sample_tokens(T) if tokens is None else np.asarray(tokens, np.int64)
    tie_toks = np.nonzero(rc.tie)[0]
    toks = np.union1d(toks, tie_toks).astype(np.int64)
    yo = c.outputs(toks, rc.ids_safe, rc.w_ref)
    yg = to_np(y_gpu).astype(np.float64)[toks]
    err = float(np.max(np.abs(yg - yo)) / max(np.max(np.abs(yo)), 1e-30)) if len(toks) else 0.0
    rep = Report(T, int(rc.tie.sum()), int(np.sum(~rc.same_set & rc.tie)),
                 int(np.isin(tie_toks, toks).sum()), rc.mismatch, rc.invalid, rc.weight_max_rel,
                 err, len(toks), rc.swaps)
    print(rep.line())
    return rep


def release(layer: Layer):
    """Drop the oracle cache (it refers back to the layer) and free the
    layer's device memory before the next module allocates its own."""
    import gc
    layer.cache = None
    gc.collect()
    torch.cuda.empty_cache()


def check(rep: Report, fmt: str = "bf16", min_compared: Optional[int] = None):
    """The acceptance rule on a Report."""
    assert rep.id_mismatch_outside_ties == 0, rep
    assert rep.invalid_tie_choices == 0, rep
    assert rep.weight_max_rel < 1e-5, rep
    assert rep.y_rel_err <= TOL[fmt], rep
    assert rep.near_tie_compared == rep.near_ties, rep  # every near-tie token's output
    want = min(rep.T, N_SAMPLE) if min_compared is None else min_compared
    assert rep.compared_tokens >= want, rep


def check_permutation(ids: np.ndarray, offsets: np.ndarray, pair_rows: np.ndarray) -> str:
    """The dispatch's row order (grouped by expert) against the routing:
    offsets are the exclusive scan of the per-expert counts (empty experts
    have offsets[e] = offsets[e+1]); pair_rows is a bijection of the T*k
    (token, slot) pairs onto [0, T*k); each pair's row lies in its expert's
    range; and within an expert the rows are in ascending token order."""
    ids = np.asarray(ids, np.int64)
    T, k = ids.shape
    E = len(offsets) - 1
    offsets = np.asarray(offsets, np.int64)
    pr = np.asarray(pair_rows, np.int64).ravel()
    counts = np.bincount(ids.ravel(), minlength=E)
    assert offsets[0] == 0 and offsets[E] == T * k, (offsets[0], offsets[E])
    assert np.array_equal(np.diff(offsets), counts), "offsets are not the scan of the counts"
    assert np.array_equal(np.sort(pr), np.arange(T * k)), "pair rows are not a bijection"
    owner = np.repeat(np.arange(E), counts)  # expert of each row
    assert np.array_equal(owner[pr], ids.ravel()), "a pair's row is outside its expert's range"
    tok_of_row = np.empty(T * k, np.int64)
    tok_of_row[pr] = np.repeat(np.arange(T), k)
    same_expert = owner[1:] == owner[:-1]
    assert np.all(np.diff(tok_of_row)[same_expert] > 0), "rows of an expert not in token order"
    return (f"permutation of {T * k} pairs over {E} experts: bijective, grouped, token order; "
            f"{int((counts == 0).sum())} empty experts, largest {int(counts.max())} rows")
