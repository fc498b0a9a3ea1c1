"""Host logic of bench.py without a GPU: the multi-rank aggregation (max of
the per-rank step time, sum of tokens) over a 2-rank gloo group, the
workload table, and the algorithmic byte/flop counts."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synth


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        ms, tok = bench.aggregate_over_ranks(1.0 + rank * 2.5, 64, torch.device("cpu"))
        bench.barrier(torch.device("cpu"))
        out[rank] = (ms, tok)
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1] == (3.5, 128)


def test_single_rank_is_identity():
    assert bench.aggregate_over_ranks(2.0, 64, torch.device("cpu")) == (2.0, 64)


def test_workloads():
    assert bench.workload("decode")["T"] == 64
    assert bench.workload("prefill")["T"] == 8192
    w = bench.workload("fp8-T1024")
    assert w["T"] == 1024 and w["fmt"] == "fp8"
    with pytest.raises(SystemExit):
        bench.workload("nope")


def test_algorithmic_counts_match_the_expert_size():
    # every expert hit once: the weight bytes are (E + 1) experts x 3 matrices
    s = synth.K2
    ids = np.arange(384).reshape(48, 8)
    a = bench.algorithmic(s, 48, "bf16", ids)
    assert a["U"] == 384
    per_expert = 3 * 7168 * 2048 * 2  # BF16: 88,080,384 bytes per expert
    assert per_expert == 88080384
    assert a["layer"][0] - (385 * per_expert) == 384 * 7168 * 4 + 384 * 4 + 48 * 7168 * 4
    R = 48 * 9
    assert a["gemm_gate_up"][1] == 2 * R * 2 * 2048 * 7168


def test_dense_workload_and_its_counts():
    """K2's dense FFN layer: no router, 9 shared groups of 2048 (intermediate
    18432); its algorithmic work is one 3 x 7168 x 18432 MLP over T rows."""
    w = bench.workload("dense-T64")
    s = w["shape"]
    assert (w["T"], w["fmt"]) == (64, "bf16")
    assert (s.n_routed_experts, s.num_experts_per_tok, s.n_shared_experts) == (0, 0, 9)
    assert s.moe_intermediate_size * s.n_shared_experts == 18432
    assert bench.workload("dense-fp8-T128")["fmt"] == "fp8"
    T = 64
    a = bench.algorithmic(s, T, "bf16", np.zeros((T, 0), np.int64))
    assert a["U"] == 0
    # gate/up: the weights once, x once per token (not per gathered row), h
    # once per row
    assert a["gemm_gate_up"][0] == 2 * 18432 * 7168 * 2 + T * 7168 * 2 + T * 9 * 2048 * 2
    assert a["gemm_gate_up"][1] == 2 * T * 2 * 18432 * 7168
    assert a["gemm_down"][1] == 2 * T * 18432 * 7168
    # down: the weights once, h rows in, BF16 per-row outputs out
    assert a["gemm_down"][0] == 18432 * 7168 * 2 + T * 9 * 2048 * 2 + T * 9 * 7168 * 2
    assert a["layer"][1] == 2 * T * 3 * 18432 * 7168


def test_reference_arm_prints_the_contract_line(capsys):
    """`bench.py --impl reference` (the float64 oracle on the host cores) prints
    one JSON line with the bench keys, impl "reference", a cpu_baseline of
    kind "oracle" equal to the line's value, and an e2e that moves no bytes."""
    import json
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--tokens", "8",
                "--experts", "16"])
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in j, key
    assert j["impl"] == "reference" and j["dtype"] == "f64" and j["n_gpus"] == 1
    assert j["steps"] == 1 and j["warmup"] == 0 and j["higher_is_better"] is True
    assert j["value"] > 0 and j["unit"] == "tokens/s"
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
    assert "tokens" in cb["sample"]
    e2e = j["e2e"]
    assert e2e["value"] == j["value"] and e2e["unit"] == j["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert j["config"]["tokens"] == 8 and j["config"]["n_routed_experts"] == 16


def test_traffic_only_for_the_workload_it_was_taken_on(tmp_path, monkeypatch):
    # a committed traffic figure counts only for its own full-size workload and
    # only while the GEMM sources it was measured on are unchanged
    src = bench.kernel_src_hash("gemm_gate_up")
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(
        '{"decode": {"gemm_gate_up": {"bytes_per_launch": 123, "src": "%s"}},'
        ' "prefill": {"gemm_gate_up": {"bytes_per_launch": 456, "src": "stale"}}}' % src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_src_hash", lambda k: src)
    assert bench.traffic_for("gemm_gate_up", "decode") == 123
    assert bench.traffic_for("gemm_gate_up", "prefill") is None  # sources changed since
    assert bench.traffic_for("gemm_gate_up", None) is None  # a reduced case
    assert bench.traffic_for("gemm_down", "decode") is None


def test_clock_sampler_follows_cuda_visible_devices(monkeypatch):
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    assert bench.smi_device(1) == "1"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "5,3")
    assert bench.smi_device(0) == "5" and bench.smi_device(1) == "3"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-aaaa")
    assert bench.smi_device(0) == "GPU-aaaa"
