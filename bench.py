"""Throughput of the K2 routed-MoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl native|reference]

One step = one forward of the whole layer (router, top-8, dispatch, gate/up
GEMM + SwiGLU, down GEMM, weighted combine with the shared expert) over one
batch of T synthetic tokens with weights resident in HBM. Prints one JSON
line (rank 0).

Workloads (--config):
  decode      K2 layer, T = 64 tokens, BF16 experts (default); the line also
              carries a "prefill" key: the same measurement at T = 8192 on
              the same weights and handle (--no-prefill leaves it out)
  prefill     K2 layer, T = 8192 tokens, BF16 experts
  fp8-T<n>    K2 layer, T = n tokens, FP8 e4m3 experts with 128x128 scales
  dense-T<n>  K2's dense FFN layer (its first layer: one SwiGLU MLP of
              intermediate 18432, no router), T = n tokens, BF16 (dense-fp8-T<n>: FP8)

N > 1 runs one independent replica per GPU (data parallel over token
batches; the layer has no exchange step at one GPU per replica), so the
scaling is weak and the value is the tokens of all ranks / the slowest rank's
time. Timing: CUDA events on the launch stream, W warm-up steps, then K
plain forwards (as a caller runs them) between a barrier + synchronize on
both sides; max over ranks. The phase times and the dominant kernel's
roofline come from a further run of the same forwards with the library's
per-phase events. The
weights streamed per step (25-34 GB BF16) are far larger than the 126 MB L2,
so no flush is needed between steps.

--impl reference times the CPU oracle (float64 numpy) on the host cores, on
a bounded sample of the same workload each step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "K2 MoE layer tokens/s; % of HBM (decode) / tensor-peak (prefill) roofline"
PREFILL_T = 8192
UNIT = "tokens/s"
PHASES = ("router_logits", "router_topk", "route_scan", "dispatch", "gemm_gate_up",
          "gemm_down", "combine")
_GEMM_SOURCES = ["gemm_bf16.cu", "gemm_bf16_2sm.cu", "gemm_promoted.cu", "gemm_common.cuh",
                 "sm100.cuh", "dispatch.cu"]
KERNEL_SOURCES = {"gemm_gate_up": _GEMM_SOURCES, "gemm_down": _GEMM_SOURCES}


# ----------------------------------------------------------------- workloads
def workload(name: str):
    if name == "decode":
        return dict(T=64, fmt="bf16", with_prefill=True,
                    desc="K2 MoE layer decode step, T=64 tokens, BF16 experts")
    if name == "prefill":
        return dict(T=8192, fmt="bf16", desc="K2 MoE layer prefill, T=8192 tokens, BF16 experts")
    if name.startswith("dense-"):
        fmt = "fp8" if name.startswith("dense-fp8-T") else "bf16"
        T = int(name.split("T")[-1])
        shape = synth.LayerShape(n_routed_experts=0, num_experts_per_tok=0, n_shared_experts=9)
        return dict(T=T, fmt=fmt, shape=shape,
                    desc=f"K2 dense FFN layer (intermediate 18432 = 9 x 2048, no router), "
                         f"T={T} tokens, {fmt.upper()} weights")
    if name.startswith("fp8-T"):
        T = int(name[5:])
        return dict(T=T, fmt="fp8", desc=f"K2 MoE layer, T={T} tokens, FP8 e4m3 experts "
                                           "(128x128 block scales, dynamic activation quant)")
    raise SystemExit(f"unknown --config {name}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm=j["hbm_gbs"], bf16=j["bf16_tflops"], bf16_sus=j["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ------------------------------------------------------- distributed helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate_over_ranks(ms: float, tokens: int, device) -> tuple:
    """(max over ranks of ms, sum over ranks of tokens); identity at world size 1."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms, tokens
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    n = torch.tensor([tokens], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return float(t.item()), int(n.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.zeros(1, device=device)
        dist.all_reduce(t)


# ------------------------------------------------------------------- clocks
def smi_device(local: int) -> str:
    """The nvidia-smi id (-i) of CUDA device `local`: CUDA_VISIBLE_DEVICES
    renumbers devices, nvidia-smi does not (it takes the listed index or UUID)."""
    vis = [v.strip() for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v.strip()]
    return vis[local] if local < len(vis) else str(local)


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    Q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            p = [s.strip() for s in ln.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx = float(p[1])
            except ValueError:
                continue
            for n, v in zip(names, p[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- CPU baseline
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


class OracleSample:
    """The CPU oracle on a bounded sample of the workload: routing of all T
    tokens (or of the sample when T is large) and the experts of `n_tok`
    sampled tokens, with their weights already on the host."""

    def __init__(self, shape, T, fmt, n_tok, x_cpu, Wg_cpu, b_cpu, fetch_expert, seed=7):
        from oracle import moe as orc
        self.orc, self.shape, self.fmt = orc, shape, fmt
        rng = np.random.default_rng(seed)
        self.T = T
        self.route_rows = min(T, 256)
        self.x = x_cpu.float().numpy().astype(np.float64)
        self.Wg = Wg_cpu.numpy().astype(np.float64)
        self.b = b_cpu.numpy().astype(np.float64)
        self.tok = np.sort(rng.choice(T, size=min(n_tok, T), replace=False))
        self.shared = fetch_expert(-1) if shape.n_shared_experts > 0 else None
        self.dense = shape.n_routed_experts == 0
        if self.dense:  # no router: the shared MLP alone
            self.rows = self.tok
            return
        rows = np.union1d(self.tok, rng.choice(T, size=self.route_rows, replace=False))
        self.rows = rows
        r = orc.route(self.x[rows], self.Wg, self.b, shape.num_experts_per_tok,
                      shape.routed_scaling_factor, shape.norm_topk_prob)
        pos = np.searchsorted(rows, self.tok)
        need = sorted(set(int(e) for e in r.ids[pos].ravel()))
        self.cache = {e: fetch_expert(e) for e in need}
        self.pos = pos

    def run_once(self) -> int:
        s, orc = self.shape, self.orc
        if self.dense:
            orc.dense_ffn(self.x[self.tok], self.shared, self.fmt)
            return len(self.tok)
        r = orc.route(self.x[self.rows], self.Wg, self.b, s.num_experts_per_tok,
                      s.routed_scaling_factor, s.norm_topk_prob)
        orc.experts_combine(self.x[self.rows], r.ids, r.weights, lambda e: self.cache[e],
                            (lambda: self.shared) if self.shared is not None else None,
                            self.fmt, s.n_shared_experts, self.pos)
        return len(self.tok)

    def describe(self):
        if self.dense:
            return (f"{len(self.tok)} of {self.T} tokens through the dense FFN, weights "
                    "preloaded on the host")
        return (f"{len(self.tok)} of {self.T} tokens through the experts (routing for "
                f"{len(self.rows)} tokens), weights preloaded on the host")


def np_expert(mats: dict) -> dict:
    out = {}
    for n, v in mats.items():
        out[n] = v.numpy() if v.dtype == torch.uint8 else v.float().numpy()
    return out


# -------------------------------------------------------------------- arms
def algorithmic(shape, T, fmt, ids: np.ndarray):
    """Algorithmic bytes and flops of each GEMM launch, and of the layer, for
    the actual routing. x counts once per token (T rows, the method's input;
    the gathered copy per (token, slot) is this library's intermediate), h
    once per routed row (written by gate/up, read by down), the per-row
    outputs once per routed row (BF16, read by the combine)."""
    d, f, E, k, ns = (shape.hidden_size, shape.moe_intermediate_size, shape.n_routed_experts,
                      shape.num_experts_per_tok, shape.n_shared_experts)
    wb = 1 if fmt == "fp8" else 2
    U = len(np.unique(ids)) if E > 0 else 0
    G_used = U + ns
    R = T * (k + ns)
    sb = lambda r, c: (r // 128) * (c // 128) * 4 if fmt == "fp8" else 0
    gate_up_bytes = G_used * 2 * (f * d * wb + sb(f, d)) + T * d * wb + R * f * wb
    down_bytes = G_used * (d * f * wb + sb(d, f)) + R * f * wb + R * d * 2  # BF16 row outputs
    if fmt == "fp8":
        gate_up_bytes += T * (d // 128) * 4 + R * (f // 128) * 4
        down_bytes += R * (f // 128) * 4
    gate_up_flops = 2 * R * 2 * f * d
    down_flops = 2 * R * d * f
    layer_bytes = G_used * 3 * (d * f * wb + sb(d, f)) + E * d * 4 + E * 4 + T * d * 2 * 2
    layer_flops = 2 * R * 3 * d * f + 2 * T * E * d
    return dict(U=U, gemm_gate_up=(gate_up_bytes, gate_up_flops),
                gemm_down=(down_bytes, down_flops), layer=(layer_bytes, layer_flops))


# datasheet figures (dense, HGX B200) beside the measured ones
DATASHEET = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def kernel_src_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        p = os.path.join(ROOT, "sparse_moe_sigmoid_b200", "csrc", f)
        if os.path.exists(p):
            h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, config: str):
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    j = json.load(open(p)).get(config, {}).get(kernel)
    if not j or j.get("src") != kernel_src_hash(kernel):
        return None
    return j.get("bytes_per_launch")


def measure(smoe, h, x, y, T, fmt, shape, args, dev, config_name):
    """Time K plain forwards of T tokens (after W warm-ups), then the same
    forwards with the library's phase events, then end to end from pinned
    host memory. Returns the measurement as a dict (max over ranks)."""
    ws, rank, local = dist_env()
    stream = torch.cuda.current_stream()
    ids = torch.empty((T, max(shape.num_experts_per_tok, 1)), dtype=torch.int32, device=dev)
    if shape.n_routed_experts > 0:
        smoe.moe_forward(h, x, y, topk_ids_out=ids, flags=smoe.MOE_FLAG_SYNC_CHECK)
        ids_np = ids.cpu().numpy()
    else:
        smoe.moe_forward(h, x, y, flags=smoe.MOE_FLAG_SYNC_CHECK)
        ids_np = np.zeros((T, 0), np.int64)
    for _ in range(args.warmup):
        smoe.moe_forward(h, x, y)
    torch.cuda.synchronize()

    # the timed steps: plain forwards, as a caller runs them (the library
    # replays them as a CUDA graph from the second call on)
    n0 = smoe.moe_launch_count(h)
    clocks = ClockSampler(smi_device(local))
    clocks.start()
    time.sleep(0.3)
    barrier(dev)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        smoe.moe_forward(h, x, y)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(dev)
    clk = clocks.stop()
    launches = smoe.moe_launch_count(h) - n0
    ms_total = e0.elapsed_time(e1)
    # then the same forwards with the library's per-phase events (launched one
    # by one), for the phase times and the dominant kernel's roofline
    n_prof = min(args.steps, 50)
    smoe.moe_profile_enable(h, n_prof)
    for _ in range(n_prof):
        smoe.moe_forward(h, x, y)
    torch.cuda.synchronize()
    phases = np.array(smoe.moe_profile_read(h, n_prof))
    smoe.moe_profile_enable(h, 0)
    st = smoe.moe_get_device_status(h)
    if st:
        raise SystemExit(f"device status word set during the timed steps: {st:#x}")

    # end to end through the host-memory entry point, copies included
    xh = x.cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    for _ in range(2):
        smoe.moe_forward_host(h, xh, yh)
        smoe.moe_forward_host_async(h, xh, yh)
    smoe.moe_host_wait(h)
    n_e2e = max(3, min(args.steps, 50))
    barrier(dev)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(n_e2e):
        # every step: upload x from pinned memory, forward, download y; the
        # library overlaps each step's copies with its neighbours' forwards
        smoe.moe_forward_host_async(h, xh, yh)
    smoe.moe_host_wait(h)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / n_e2e
    e2e_ms, _ = aggregate_over_ranks(e2e_ms, T, dev)

    ms_step = ms_total / args.steps
    ms_max, tokens_all = aggregate_over_ranks(ms_step, T, dev)
    value = tokens_all / (ms_max / 1e3)

    # roofline of the dominant kernel, timed live by the library's phase events
    mean_ph = phases.mean(axis=0)
    dom = int(np.argmax(mean_ph))
    dom_name = PHASES[dom]
    alg = algorithmic(shape, T, fmt, ids_np)
    if dom_name == "gemm_gate_up" and mean_ph[PHASES.index("gemm_down")] == 0.0:
        # the single-launch layer runs both GEMMs as one pipeline (the down
        # phase is reported empty): charge the phase with both GEMMs' work
        gu_b, gu_f = alg["gemm_gate_up"]
        dn_b, dn_f = alg["gemm_down"]
        dom_name = "gemm_gate_up+down"
        alg[dom_name] = (gu_b + dn_b, gu_f + dn_f)
    peaks = load_peaks()
    ten_peak = peaks["bf16_sus"] * (2.0 if fmt == "fp8" else 1.0)
    ten_sheet = DATASHEET["bf16_tflops"] * (2.0 if fmt == "fp8" else 1.0)
    byts, flops = alg.get(dom_name, alg["layer"])
    dur = mean_ph[dom] / 1e3
    hbm_t = byts / (peaks["hbm"] * 1e9)
    ten_t = flops / (ten_peak * 1e12)
    if hbm_t >= ten_t:
        roof = {"bound": "hbm", "achieved": byts / dur / 1e9, "peak": peaks["hbm"],
                "unit": "GB/s"}
    else:
        roof = {"bound": "tensor", "achieved": flops / dur / 1e12, "peak": ten_peak,
                "unit": "TFLOP/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(dom_name, config_name)
    roof.update({
        "kernel": dom_name, "launch_ms": round(mean_ph[dom], 4),
        "algorithmic_bytes": int(byts), "algorithmic_flops": int(flops),
        "hbm_frac": (byts / dur / 1e9) / peaks["hbm"],
        "tensor_frac": (flops / dur / 1e12) / ten_peak,
        "hbm_frac_datasheet": (byts / dur / 1e9) / DATASHEET["hbm_gbs"],
        "tensor_frac_datasheet": (flops / dur / 1e12) / ten_sheet,
        "peak_source": f"{peaks['src']} (HBM copy GB/s; sustained cuBLAS bf16 TF/s"
                       f"{', x2 nominal fp8 ratio' if fmt == 'fp8' else ''}); the *_datasheet "
                       f"fractions use 8 TB/s and {ten_sheet:.0f} TF/s dense"})
    layer_bytes, layer_flops = alg["layer"]
    sec = ms_max / 1e3
    return {
        "T": T, "value": value, "ms_per_step": ms_max, "U": alg["U"],
        "roofline": roof,
        "layer_roofline": {
            "bytes": int(layer_bytes), "flops": int(layer_flops),
            "hbm_frac": (layer_bytes / sec / 1e9) / peaks["hbm"],
            "tensor_frac": (layer_flops / sec / 1e12) / ten_peak,
            "hbm_frac_datasheet": (layer_bytes / sec / 1e9) / DATASHEET["hbm_gbs"],
            "tensor_frac_datasheet": (layer_flops / sec / 1e12) / ten_sheet},
        "phases_ms": {p: round(float(v), 4) for p, v in zip(PHASES, mean_ph)},
        "e2e": {"value": tokens_all / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": int(xh.numel() * 2),
                "d2h_bytes_per_step": int(yh.numel() * 2), "ms_per_step": e2e_ms,
                "api": "moe_forward_host_async + moe_host_wait (pinned host x and y; uploads "
                       "and downloads overlap neighbouring forwards)"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }


def run_native(args, wl):
    import sparse_moe_sigmoid_b200 as smoe
    ws, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    shape, T, fmt = wl.get("shape", synth.K2), wl["T"], wl["fmt"]
    # the default (decode) line also measures prefill on the same weights
    T_pre = PREFILL_T if (wl.get("with_prefill") and not args.no_prefill) else 0
    T_max = max(T, T_pre)
    x_all = synth.make_tokens(shape, T_max, device=dev)
    x = x_all[:T].contiguous()
    Wg, b = synth.make_router(shape, device=dev)
    ew = synth.make_experts(shape, device=dev, fmt=fmt)
    cfg = smoe.moe_config_init_k2(
        max_tokens=T_max, n_routed_experts=shape.n_routed_experts,
        single_launch_max_tokens=args.single_launch_max_tokens,
        num_experts_per_tok=shape.num_experts_per_tok, n_shared_experts=shape.n_shared_experts,
        weight_format=smoe.MOE_WEIGHT_BF16 if fmt == "bf16" else smoe.MOE_WEIGHT_FP8_E4M3_BLOCK)
    h = smoe.moe_create(cfg, local)
    smoe.moe_load_weights(h, Wg, b, ew.gate, ew.up, ew.down, ew.shared_gate, ew.shared_up,
                          ew.shared_down, ew.gate_scale, ew.up_scale, ew.down_scale,
                          ew.shared_gate_scale, ew.shared_up_scale, ew.shared_down_scale)
    torch.cuda.synchronize()

    # CPU oracle baseline (rank 0, one GPU only), before the caller copies go
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        n_tok = 4 if T <= 64 else 3
        ors = OracleSample(shape, T, fmt, n_tok, x.cpu(), Wg.cpu(), b.cpu(),
                           lambda e: np_expert(synth.expert_slice(ew, e) if e >= 0
                                               else synth.shared_slice(ew)))
        t0 = time.perf_counter()
        n, reps = 0, 0
        while True:
            n += ors.run_once()
            reps += 1
            if time.perf_counter() - t0 > 10.0 or reps >= 20:
                break
        el = time.perf_counter() - t0
        cpu = {"value": n / el, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{ors.describe()}; {reps} repetitions in {el:.1f} s"}
    del ew
    torch.cuda.empty_cache()

    y = torch.empty_like(x)
    # DRAM traffic figures belong to the full-size workloads they were taken on
    traffic_key = None if wl.get("reduced") else args.config
    m = measure(smoe, h, x, y, T, fmt, shape, args, dev, traffic_key)
    pre = None
    if T_pre:
        xp = x_all[:T_pre].contiguous()
        pre = measure(smoe, h, xp, torch.empty_like(xp), T_pre, fmt, shape, args, dev,
                      None if wl.get("reduced") else "prefill")
        pre = {"workload": f"K2 MoE layer prefill, T={T_pre} tokens, {fmt.upper()} experts "
                           "(same weights and handle)",
               "ms_per_step": pre["ms_per_step"], "value": pre["value"], "unit": UNIT,
               "roofline": pre["roofline"], "layer_roofline": pre["layer_roofline"],
               "phases_ms": pre["phases_ms"], "e2e": pre["e2e"],
               "gpu_launches": pre["gpu_launches"], "clocks": pre["clocks"],
               "distinct_experts_hit": pre["U"]}
    out = {
        "metric": METRIC, "value": m["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if fmt == "bf16" else "e4m3",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights, random init)",
        "config": {"workload": wl["desc"], "tokens": T, "global_batch": T * ws,
                   "hidden_size": shape.hidden_size, "n_routed_experts": shape.n_routed_experts,
                   "top_k": shape.num_experts_per_tok, "n_shared_experts": shape.n_shared_experts,
                   "moe_intermediate_size": shape.moe_intermediate_size,
                   "parallelism": f"replicas x{ws}", "distinct_experts_hit": m["U"],
                   "single_launch_max_tokens": args.single_launch_max_tokens,
                   "l2": "no flush: the expert weights streamed each step exceed the 126 MB L2"},
        "roofline": m["roofline"],
        "layer_roofline": m["layer_roofline"],
        "phases_ms": m["phases_ms"],
        "cpu_baseline": cpu,
        "e2e": m["e2e"],
        "gpu_launches": m["gpu_launches"] + (pre["gpu_launches"] if pre else 0),
        "clocks": m["clocks"],
    }
    if pre:
        out["prefill"] = pre
        out["gpu_launches_note"] = ("kernels launched in the timed regions of the decode line "
                                    "and of the prefill key together")
    smoe.moe_destroy(h)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def run_reference(args, wl):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    shape, T, fmt = wl.get("shape", synth.K2), wl["T"], wl["fmt"]
    x = synth.make_tokens(shape, T)
    Wg, b = synth.make_router(shape)
    n_tok = 2
    ors = OracleSample(shape, T, fmt, n_tok, x, Wg, b,
                       lambda e: np_expert(synth.make_expert(shape, e, fmt=fmt)))
    for _ in range(args.warmup):
        ors.run_once()
    t0 = time.perf_counter()
    n = 0
    for _ in range(args.steps):
        n += ors.run_once()
    el = time.perf_counter() - t0
    value = n / el
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "impl": "reference",
        "data": "synthetic (seeded N(0,1) tokens, N(0,0.02) weights, random init)",
        "config": {"workload": wl["desc"], "tokens": T, "global_batch": T * ws,
                   "hidden_size": shape.hidden_size, "n_routed_experts": shape.n_routed_experts,
                   "top_k": shape.num_experts_per_tok, "n_shared_experts": shape.n_shared_experts,
                   "moe_intermediate_size": shape.moe_intermediate_size,
                   "parallelism": "host cores, rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"each step: {ors.describe()}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="decode")
    ap.add_argument("--impl", default="native", choices=("native", "reference"))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="decode line only (no prefill key)")
    ap.add_argument("--single-launch-max-tokens", type=int, default=0,
                    help="batches up to this size run the layer as one launch (0: never)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override T (small profiling cases)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override n_routed_experts (small profiling cases)")
    args = ap.parse_args(argv)
    wl = workload(args.config)
    if args.tokens is not None or args.experts is not None:
        wl["T"] = args.tokens or wl["T"]
        E = args.experts or synth.K2.n_routed_experts
        wl["shape"] = synth.LayerShape(n_routed_experts=E)
        wl["desc"] += f" [reduced case: T={wl['T']}, {E} routed experts]"
        wl["reduced"] = True
    if args.steps is None:
        args.steps = (400 if wl["T"] <= 1024 else 100) if args.impl == "native" else 5
    if args.warmup < 3 and args.impl == "native":
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_native(args, wl)


if __name__ == "__main__":
    main()
