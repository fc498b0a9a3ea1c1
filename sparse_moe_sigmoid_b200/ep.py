"""Expert parallelism over the GPUs of one node (EP = world size).

The pages deploy K2 with expert parallelism ("Behind Kimi-K2's Config" §2 and
§2.1: EP = 128, each rank holding its routed experts plus the shared expert;
"Kimi K2 · Down projection": the module builds only its rank's slice of the
384 experts, experts_per_rank = n_routed_experts / ep_size). Here rank r of N
owns the contiguous slice [r * E / N, (r + 1) * E / N) of the routed experts
and a replica of the router and of the shared expert. One forward over rank
r's own tokens x_r [T_r, d]:

  1. route every token over all E experts (ids [T_r, k], weights);
  2. plan: each (token, slot) pair goes to the rank owning its expert; pairs
     are ordered by destination rank, then by pair index t * k + j;
  3. dispatch: per-destination counts are exchanged, then each pair's x row
     and its expert's index inside the owner's slice;
  4. the owner runs its experts on the rows it received, one output row per
     pair, unweighted: E_e(x_t);
  5. the output rows travel back (the split sizes swapped) and are put back
     in (token, slot) order;
  6. combine: y[t] = sum_j w[t, j] * out[t, j] + S(x_t), S the shared expert
     on the rank's own tokens.

The plan is index arithmetic and the exchange is torch.distributed (NCCL
between GPUs; rows are staged in each GPU's own memory, no peer memory is
read by any kernel); routing, experts, shared expert and combine are the
library's kernels (make_library_callables).
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional

import torch
import torch.distributed as dist


@dataclasses.dataclass
class Plan:
    """Where each (token, slot) pair of this rank goes."""
    order: torch.Tensor      # [T * k] pair indices t * k + j sorted by (owner, pair index)
    send_counts: List[int]   # pairs sent to each rank (in `order`)
    local_id: torch.Tensor   # [T * k] int32 expert index inside the owner's slice, in `order`


def experts_per_rank(n_experts: int, world: int) -> int:
    """Size of each rank's contiguous slice of the routed experts."""
    if world < 1 or n_experts % world:
        raise ValueError("n_routed_experts must split evenly over the ranks")
    return n_experts // world


def make_plan(ids: torch.Tensor, n_experts: int, world: int) -> Plan:
    """ids [T, k] global expert ids -> this rank's dispatch plan. Expert e
    belongs to rank e // experts_per_rank."""
    per = experts_per_rank(n_experts, world)
    flat = ids.reshape(-1).to(torch.int64)
    if flat.numel() and (int(flat.min()) < 0 or int(flat.max()) >= n_experts):
        raise ValueError("expert id out of range")
    dest = torch.div(flat, per, rounding_mode="floor")
    n = flat.numel()
    order = torch.argsort(dest * n + torch.arange(n, device=flat.device))
    counts = torch.bincount(dest, minlength=world)
    local = (flat - dest * per)[order].to(torch.int32)
    return Plan(order, [int(c) for c in counts.tolist()], local)


def exchange_counts(send_counts: List[int], device, group=None) -> List[int]:
    """all_to_all of the per-destination counts: entry q of the result is the
    number of rows rank q sends here."""
    s = torch.tensor(send_counts, dtype=torch.int64, device=device)
    r = torch.empty_like(s)
    dist.all_to_all_single(r, s, group=group)
    return [int(v) for v in r.tolist()]


def exchange(send: torch.Tensor, send_counts: List[int], recv_counts: List[int],
             group=None) -> torch.Tensor:
    """all_to_all of the rows of `send`, grouped by destination in rank order."""
    recv = send.new_empty((sum(recv_counts),) + tuple(send.shape[1:]))
    dist.all_to_all_single(recv, send.contiguous(), recv_counts, send_counts, group=group)
    return recv


def ep_forward(x: torch.Tensor, route: Callable, experts: Callable,
               shared: Optional[Callable], combine: Callable, n_experts: int, k: int,
               group=None) -> torch.Tensor:
    """One expert-parallel forward of this rank's tokens x [T, d] (module
    docstring). route(x) -> (ids [T, k], w [T, k]); experts(rows, local_ids)
    -> this rank's expert outputs, one row per input row; shared(x) -> S(x),
    or None without a shared expert; combine(pair_out [T * k, d], w,
    shared_out) -> y [T, d]. Every rank must call it (it exchanges with all
    of them), also with no tokens."""
    world = dist.get_world_size(group)
    ids, w = route(x)
    plan = make_plan(ids, n_experts, world)
    recv_counts = exchange_counts(plan.send_counts, x.device, group)
    token_of_pair = torch.div(plan.order, k, rounding_mode="floor")
    rows_in = exchange(x.index_select(0, token_of_pair), plan.send_counts, recv_counts, group)
    local_in = exchange(plan.local_id.view(-1, 1), plan.send_counts, recv_counts,
                        group).view(-1)
    out_in = experts(rows_in, local_in)
    out_back = exchange(out_in, recv_counts, plan.send_counts, group)
    pair_out = torch.empty_like(out_back)
    pair_out.index_copy_(0, plan.order, out_back)  # back to (token, slot) order
    return combine(pair_out, w, shared(x) if shared is not None else None)


class LibraryEP:
    """One rank's share of the layer on its GPU, through the library's C ABI:
    the router (moe_router_topk_noalloc, over all experts), this rank's slice
    of the routed experts (a handle with k = 1, weight 1 and the expert forced
    per row, so each row's output is E_e(x)), the shared expert (a handle with
    no routed experts) and the combine (moe_combine_rows). FP8 weights take
    their block scales (the routed ones sliced like the weights). Group-limited
    routing (n_group > 1) is refused: the allocation-free router routes over
    all experts with n_group = 1."""

    def __init__(self, smoe, cfg, router_weight, bias, gate, up, down, shared_gate=None,
                 shared_up=None, shared_down=None, max_tokens=8192, group=None, device=None,
                 gate_scale=None, up_scale=None, down_scale=None, shared_gate_scale=None,
                 shared_up_scale=None, shared_down_scale=None):
        if cfg.n_group > 1:
            raise ValueError("expert parallelism here routes with n_group = 1; "
                             f"the config asks for n_group = {cfg.n_group}")
        fp8 = cfg.weight_format == smoe.MOE_WEIGHT_FP8_E4M3_BLOCK
        if fp8 and (gate_scale is None or up_scale is None or down_scale is None):
            raise ValueError("FP8 expert weights need their block scales")
        self.smoe, self.group = smoe, group
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        self.E, self.k = cfg.n_routed_experts, cfg.num_experts_per_tok
        self.norm, self.scale = cfg.norm_topk_prob, cfg.routed_scaling_factor
        per = experts_per_rank(self.E, world)
        lo = rank * per
        self.router_weight, self.bias = router_weight, bias
        dev = router_weight.device if device is None else device
        dev_index = dev.index if dev.index is not None else torch.cuda.current_device()
        d = cfg.hidden_size
        fmt = dict(weight_format=cfg.weight_format,
                   weight_block_size=tuple(cfg.weight_block_size))
        sl = (lambda t: None if t is None else t[lo:lo + per])
        ex_cfg = smoe.moe_config_init_k2(
            hidden_size=d, moe_intermediate_size=cfg.moe_intermediate_size,
            n_routed_experts=per, num_experts_per_tok=1, n_shared_experts=0,
            norm_topk_prob=1, routed_scaling_factor=1.0,
            max_tokens=max(1, world * max_tokens * self.k), **fmt)
        self.ex = smoe.moe_create(ex_cfg, dev_index)
        zero_w = torch.zeros((per, d), dtype=torch.float32, device=dev)  # routing is forced
        zero_b = torch.zeros((per,), dtype=torch.float32, device=dev)
        smoe.moe_load_weights(self.ex, zero_w, zero_b, sl(gate), sl(up), sl(down),
                              gate_scale=sl(gate_scale), up_scale=sl(up_scale),
                              down_scale=sl(down_scale))
        self.sh = None
        if shared_gate is not None and cfg.n_shared_experts > 0:
            sh_cfg = smoe.moe_config_init_k2(
                hidden_size=d, moe_intermediate_size=cfg.moe_intermediate_size,
                n_routed_experts=0, num_experts_per_tok=0,
                n_shared_experts=cfg.n_shared_experts, max_tokens=max(1, max_tokens), **fmt)
            self.sh = smoe.moe_create(sh_cfg, dev_index)
            smoe.moe_load_weights(self.sh, None, None, None, None, None, shared_gate, shared_up,
                                  shared_down, shared_gate_scale=shared_gate_scale,
                                  shared_up_scale=shared_up_scale,
                                  shared_down_scale=shared_down_scale)
        torch.cuda.synchronize(dev)

    def route(self, x):
        T = x.shape[0]
        ids = torch.empty((T, self.k), dtype=torch.int32, device=x.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=x.device)
        if T:
            self.smoe.moe_router_topk_noalloc(x, self.router_weight, self.bias, self.k, ids, w,
                                              norm_topk_prob=self.norm,
                                              routed_scaling_factor=self.scale)
        return ids, w

    def experts(self, rows, local_ids):
        out = torch.empty_like(rows)
        if rows.shape[0]:
            self.smoe.moe_forward(self.ex, rows, out,
                                  forced_topk_ids=local_ids.view(-1, 1).contiguous())
        return out

    def shared(self, x):
        if self.sh is None:
            return None
        out = torch.empty_like(x)
        if x.shape[0]:
            self.smoe.moe_forward(self.sh, x, out)
        return out

    def combine(self, pair_out, w, shared_out):
        T = w.shape[0]
        y = torch.empty((T, pair_out.shape[1]), dtype=pair_out.dtype, device=pair_out.device)
        if T:
            self.smoe.moe_combine_rows(pair_out, w, shared_out, y)
        return y

    def forward(self, x):
        return ep_forward(x, self.route, self.experts,
                          self.shared if self.sh is not None else None, self.combine, self.E,
                          self.k, self.group)

    def close(self):
        self.smoe.moe_destroy(self.ex)
        if self.sh is not None:
            self.smoe.moe_destroy(self.sh)
