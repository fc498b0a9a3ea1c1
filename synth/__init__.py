"""Seeded synthetic inputs for the K2 routed-MoE layer.

This module only draws random tensors of the right shapes and distributions.
It holds none of the layer's arithmetic (no routing, no expert MLP, no
activation quantisation): both the CUDA path and the CPU oracle consume what
it produces, and neither may import the other.

Shapes follow the K2 config fields (hidden_size 7168, moe_intermediate_size
2048, n_routed_experts 384, n_shared_experts 1: "Kimi K2 Base" and "Kimi K2
0905" model cards, raw config field tables) and the [out, in] weight layout
("Kimi K2 · Down projection", OpenModelAtlas, parameter accounting).
Distributions: weights ~N(0, initializer_range = 0.02), router weight fp32,
correction bias ~N(0, 0.01), inputs ~N(0, 1) in BF16.

Every tensor is drawn from its own torch generator seeded by
(seed, tensor id, expert), so a single expert can be regenerated on its own.
The same seed yields the same values on the same device type; CPU and CUDA
generators differ, so a test always hands the materialised tensors to both
sides rather than regenerating them.

FP8 checkpoints are produced the way the K2 checkpoint's quantization_config
describes them ("Kimi K2 · Down projection", config.json excerpt: fmt e4m3,
weight_block_size [128, 128]): one fp32 scale s = amax/448 per 128x128 block,
codes = e4m3(W / s) via torch's float8_e4m3fn cast. This is checkpoint
preparation, not part of the forward pass.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

SEED = 0x4B32

# tensor ids mixed into the per-tensor seeds
_TID = {"x": 1, "router": 2, "bias": 3, "gate": 4, "up": 5, "down": 6,
        "shared_gate": 7, "shared_up": 8, "shared_down": 9}


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Sizes of one MoE layer, named after the config.json fields."""
    hidden_size: int = 7168
    moe_intermediate_size: int = 2048
    n_routed_experts: int = 384
    num_experts_per_tok: int = 8
    n_shared_experts: int = 1
    routed_scaling_factor: float = 2.827
    norm_topk_prob: bool = True
    n_group: int = 1
    topk_group: int = 1


K2 = LayerShape()
TINY = LayerShape(hidden_size=256, moe_intermediate_size=128, n_routed_experts=16,
                  num_experts_per_tok=4, n_shared_experts=1)


def tensor_seed(seed: int, tensor: str, expert: int = 0) -> int:
    """64-bit seed for one tensor (splitmix64 finaliser of the mixed key)."""
    z = (seed ^ (_TID[tensor] << 48) ^ ((expert + 1) << 24)) & 0xFFFFFFFFFFFFFFFF
    z = (z + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
    z = z ^ (z >> 31)
    return z & 0x7FFFFFFFFFFFFFFF


def _randn(shape, seed: int, tensor: str, expert: int, device, std: float) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, tensor, expert))
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def make_tokens(shape: LayerShape, T: int, seed: int = SEED, device="cpu") -> torch.Tensor:
    """x: BF16 [T, hidden] ~ N(0, 1) (stands in for the RMSNorm output)."""
    return _randn((T, shape.hidden_size), seed, "x", 0, device, 1.0).to(torch.bfloat16)


def make_router(shape: LayerShape, seed: int = SEED, device="cpu", bias_std: float = 0.01,
                row_scale: Optional[torch.Tensor] = None):
    """Router weight fp32 [E, hidden] ~ N(0, 0.02) and e_score_correction_bias fp32 [E].

    row_scale (optional, [E]) multiplies each router row; it is how the skewed
    routing workload shapes expert popularity.
    """
    E, d = shape.n_routed_experts, shape.hidden_size
    w = _randn((E, d), seed, "router", 0, device, 0.02)
    if row_scale is not None:
        w.mul_(row_scale.to(device=device, dtype=torch.float32).view(E, 1))
    b = _randn((E,), seed, "bias", 0, device, bias_std)
    return w, b


def _expert_matrix(shape_rc, seed, tensor, expert, device):
    return _randn(shape_rc, seed, tensor, expert, device, 0.02)


def quantize_blocks_e4m3(w: torch.Tensor, block: int = 128):
    """Checkpoint-style FP8: per 128x128 block scale s = amax/448, codes = e4m3(w/s).

    Returns (codes uint8 [..., R, C], scales fp32 [..., R/block, C/block]).
    """
    *lead, R, C = w.shape
    wb = w.reshape(*lead, R // block, block, C // block, block)
    amax = wb.abs().amax(dim=(-3, -1))
    s = amax / 448.0
    s = torch.where(s > 0, s, torch.ones_like(s))
    q = (wb / s.unsqueeze(-2).unsqueeze(-1)).reshape(*lead, R, C)
    codes = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, s.contiguous()


@dataclasses.dataclass
class ExpertWeights:
    """Expert weights in the layout the C ABI takes ([out, in], row-major).

    BF16: gate/up [E, f, d], down [E, d, f]; shared_* are [f_s, d], [f_s, d], [d, f_s].
    FP8:  the same shapes as uint8 e4m3 codes, plus fp32 block scales
          gate_scale/up_scale [E, f/128, d/128], down_scale [E, d/128, f/128].
    """
    fmt: str
    gate: torch.Tensor
    up: torch.Tensor
    down: torch.Tensor
    shared_gate: Optional[torch.Tensor]
    shared_up: Optional[torch.Tensor]
    shared_down: Optional[torch.Tensor]
    gate_scale: Optional[torch.Tensor] = None
    up_scale: Optional[torch.Tensor] = None
    down_scale: Optional[torch.Tensor] = None
    shared_gate_scale: Optional[torch.Tensor] = None
    shared_up_scale: Optional[torch.Tensor] = None
    shared_down_scale: Optional[torch.Tensor] = None


def make_experts(shape: LayerShape, seed: int = SEED, device="cpu", fmt: str = "bf16",
                 identical: bool = False, shared_zero: bool = False) -> ExpertWeights:
    """Draw all routed + shared expert weights, expert by expert.

    identical=True reuses expert 0's draw for every routed expert (and, unless
    shared_zero, for the shared expert): the closed-form workload.
    shared_zero=True makes the shared expert's weights zero.
    """
    assert fmt in ("bf16", "fp8")
    E, d, f = shape.n_routed_experts, shape.hidden_size, shape.moe_intermediate_size
    fs = f * shape.n_shared_experts
    wdt = torch.bfloat16 if fmt == "bf16" else torch.uint8
    gate = torch.empty((E, f, d), dtype=wdt, device=device)
    up = torch.empty((E, f, d), dtype=wdt, device=device)
    down = torch.empty((E, d, f), dtype=wdt, device=device)
    scales = {}
    if fmt == "fp8":
        for n, (r, c) in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f))):
            scales[n] = torch.empty((E, r // 128, c // 128), dtype=torch.float32, device=device)
    dst = {"gate": gate, "up": up, "down": down}
    for e in range(E):
        src_e = 0 if identical else e
        for n, rc in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f))):
            w = _expert_matrix(rc, seed, n, src_e, device)
            if fmt == "bf16":
                dst[n][e].copy_(w.to(torch.bfloat16))
            else:
                q, s = quantize_blocks_e4m3(w)
                dst[n][e].copy_(q)
                scales[n][e].copy_(s)
            del w
    sh = {}
    if shape.n_shared_experts > 0:
        for n, base, rc in (("shared_gate", "gate", (fs, d)), ("shared_up", "up", (fs, d)),
                            ("shared_down", "down", (d, fs))):
            if shared_zero:
                w = torch.zeros(rc, dtype=torch.float32, device=device)
            elif identical:
                assert shape.n_shared_experts == 1
                w = _expert_matrix(rc, seed, base, 0, device)
            else:
                w = _expert_matrix(rc, seed, n, 0, device)
            if fmt == "bf16":
                sh[n] = w.to(torch.bfloat16)
            else:
                sh[n], sh[n + "_scale"] = quantize_blocks_e4m3(w)
            del w
    ew = ExpertWeights(fmt=fmt, gate=gate, up=up, down=down,
                       shared_gate=sh.get("shared_gate"), shared_up=sh.get("shared_up"),
                       shared_down=sh.get("shared_down"))
    if fmt == "fp8":
        ew.gate_scale, ew.up_scale, ew.down_scale = scales["gate"], scales["up"], scales["down"]
        ew.shared_gate_scale = sh.get("shared_gate_scale")
        ew.shared_up_scale = sh.get("shared_up_scale")
        ew.shared_down_scale = sh.get("shared_down_scale")
    return ew


def expert_slice(ew: ExpertWeights, e: int):
    """Host (CPU) copies of routed expert e's three matrices (and FP8 scales)."""
    out = {"gate": ew.gate[e].cpu(), "up": ew.up[e].cpu(), "down": ew.down[e].cpu()}
    if ew.fmt == "fp8":
        out.update(gate_scale=ew.gate_scale[e].cpu(), up_scale=ew.up_scale[e].cpu(),
                   down_scale=ew.down_scale[e].cpu())
    return out


def shared_slice(ew: ExpertWeights):
    """Host copies of the shared expert's three matrices (and FP8 scales)."""
    out = {"gate": ew.shared_gate.cpu(), "up": ew.shared_up.cpu(), "down": ew.shared_down.cpu()}
    if ew.fmt == "fp8":
        out.update(gate_scale=ew.shared_gate_scale.cpu(), up_scale=ew.shared_up_scale.cpu(),
                   down_scale=ew.shared_down_scale.cpu())
    return out


def make_expert(shape: LayerShape, e: int, seed: int = SEED, device="cpu", fmt: str = "bf16"):
    """One routed expert's matrices alone (e < E), or the shared expert (e = -1),
    drawn exactly as make_experts draws them on the same device type.
    Returns {"gate", "up", "down"} (+ "*_scale" for FP8)."""
    d, f = shape.hidden_size, shape.moe_intermediate_size
    out = {}
    for n, rc in (("gate", (f, d)), ("up", (f, d)), ("down", (d, f))):
        if e < 0:
            fs = f * shape.n_shared_experts
            rc = (fs, d) if n != "down" else (d, fs)
            w = _expert_matrix(rc, seed, "shared_" + n, 0, device)
        else:
            w = _expert_matrix(rc, seed, n, e, device)
        if fmt == "bf16":
            out[n] = w.to(torch.bfloat16)
        else:
            out[n], out[n + "_scale"] = quantize_blocks_e4m3(w)
    return out
