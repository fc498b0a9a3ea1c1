"""Python binding of the K2 routed-MoE layer library (libsmoe_b200.so).

Argument marshalling only: every function here forwards to the C entry point
of the same name in include/moe.h; all compute runs in the library's CUDA
kernels. Tensors are torch tensors (device memory and streams come from
PyTorch); they are passed as raw pointers. If the library has not been built
this module raises ImportError on import: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmoe_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sparse_moe_sigmoid_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

# ---------------------------------------------------------------- constants
MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_OOM = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE = -5
MOE_ERR_TIMEOUT = -6
MOE_ERR_STATE = -7
MOE_WEIGHT_BF16 = 0
MOE_WEIGHT_FP8_E4M3_BLOCK = 1
MOE_SCORING_SIGMOID = 0
MOE_TOPK_NOAUX_TC = 0
MOE_ACTIVATION_DYNAMIC = 0
MOE_FLAG_SYNC_CHECK = 0x1
MOE_FLAG_TEST_STALL = 0x2
MOE_FLAG_PHASE_KERNELS = 0x4
MOE_DEVICE_WAIT_TIMEOUT = 0x1
MOE_DEVICE_BAD_EXPERT_ID = 0x2
MOE_NUM_PHASES = 7
PHASES = ("router_logits", "router_topk", "route_scan", "dispatch", "gemm_gate_up",
          "gemm_down", "combine")


class moe_config_t(ctypes.Structure):
    _fields_ = [("hidden_size", ctypes.c_int32), ("moe_intermediate_size", ctypes.c_int32),
                ("n_routed_experts", ctypes.c_int32), ("num_experts_per_tok", ctypes.c_int32),
                ("n_shared_experts", ctypes.c_int32), ("n_group", ctypes.c_int32),
                ("topk_group", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("scoring_func", ctypes.c_int32),
                ("topk_method", ctypes.c_int32), ("weight_format", ctypes.c_int32),
                ("weight_block_size", ctypes.c_int32 * 2), ("activation_scheme", ctypes.c_int32),
                ("max_tokens", ctypes.c_int64), ("single_launch_max_tokens", ctypes.c_int64)]


class moe_weights_t(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_weight", "e_score_correction_bias", "gate_proj", "up_proj", "down_proj",
        "gate_scale", "up_scale", "down_scale", "shared_gate_proj", "shared_up_proj",
        "shared_down_proj", "shared_gate_scale", "shared_up_scale", "shared_down_scale")]


class moe_forward_opts_t(ctypes.Structure):
    _fields_ = [("topk_ids_out", ctypes.c_void_p), ("topk_weights_out", ctypes.c_void_p),
                ("forced_topk_ids", ctypes.c_void_p), ("router_logits_out", ctypes.c_void_p),
                ("flags", ctypes.c_uint32), ("reserved", ctypes.c_uint32),
                ("expert_offsets_out", ctypes.c_void_p), ("pair_rows_out", ctypes.c_void_p),
                ("wait_limit_ns", ctypes.c_uint64)]


_H = ctypes.c_void_p
_S = ctypes.c_int
_sig = {
    "moe_config_init_k2": (_S, [ctypes.POINTER(moe_config_t)]),
    "moe_create": (_S, [ctypes.POINTER(moe_config_t), ctypes.c_int, ctypes.POINTER(_H)]),
    "moe_load_weights": (_S, [_H, ctypes.POINTER(moe_weights_t), ctypes.c_void_p]),
    "moe_forward": (_S, [_H, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                         ctypes.POINTER(moe_forward_opts_t), ctypes.c_void_p]),
    "moe_forward_host": (_S, [_H, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                              ctypes.POINTER(moe_forward_opts_t), ctypes.c_void_p]),
    "moe_forward_host_async": (_S, [_H, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.POINTER(moe_forward_opts_t), ctypes.c_void_p]),
    "moe_host_wait": (_S, [_H]),
    "moe_get_device_status": (_S, [_H, ctypes.POINTER(ctypes.c_uint32)]),
    "moe_profile_enable": (_S, [_H, ctypes.c_int32]),
    "moe_profile_read": (_S, [_H, ctypes.POINTER(ctypes.c_float), ctypes.c_int32,
                              ctypes.POINTER(ctypes.c_int32)]),
    "moe_router_topk_noalloc": (_S, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_act_quant_e4m3": (_S, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_void_p]),
    "moe_combine_rows": (_S, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                              ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]),
    "moe_launch_count": (ctypes.c_int64, [_H]),
    "moe_destroy": (None, [_H]),
    "moe_status_string": (ctypes.c_char_p, [_S]),
    "moe_last_error": (ctypes.c_char_p, [_H]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_sig)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        msg = f"{where}: {moe_status_string(status)} ({status})"
        if detail:
            msg += f": {detail}"
        super().__init__(msg)
        self.status = status


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr() if hasattr(t, "data_ptr") else int(t)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(st: int, where: str, h=None):
    if st != MOE_OK:
        detail = _lib.moe_last_error(h).decode() if h else ""
        raise MoeError(st, where, detail)


def moe_status_string(status: int) -> str:
    return _lib.moe_status_string(status).decode()


def moe_last_error(h) -> str:
    return _lib.moe_last_error(h).decode()


def moe_config_init_k2(**overrides) -> moe_config_t:
    """The K2 layer config; keyword arguments override single fields."""
    c = moe_config_t()
    _check(_lib.moe_config_init_k2(ctypes.byref(c)), "moe_config_init_k2")
    for k, v in overrides.items():
        if k == "weight_block_size":
            c.weight_block_size[0], c.weight_block_size[1] = v
        else:
            setattr(c, k, v)
    return c


def moe_create(cfg: moe_config_t, device: int = 0):
    h = _H()
    _check(_lib.moe_create(ctypes.byref(cfg), device, ctypes.byref(h)), "moe_create")
    return h


def moe_load_weights(h, router_weight, e_score_correction_bias, gate_proj, up_proj, down_proj,
                     shared_gate_proj=None, shared_up_proj=None, shared_down_proj=None,
                     gate_scale=None, up_scale=None, down_scale=None, shared_gate_scale=None,
                     shared_up_scale=None, shared_down_scale=None, stream=None):
    w = moe_weights_t(
        _ptr(router_weight), _ptr(e_score_correction_bias), _ptr(gate_proj), _ptr(up_proj),
        _ptr(down_proj), _ptr(gate_scale), _ptr(up_scale), _ptr(down_scale),
        _ptr(shared_gate_proj), _ptr(shared_up_proj), _ptr(shared_down_proj),
        _ptr(shared_gate_scale), _ptr(shared_up_scale), _ptr(shared_down_scale))
    _check(_lib.moe_load_weights(h, ctypes.byref(w), _stream(stream)), "moe_load_weights", h)


def _opts(topk_ids_out=None, topk_weights_out=None, forced_topk_ids=None,
          router_logits_out=None, flags=0, expert_offsets_out=None, pair_rows_out=None,
          wait_limit_ns=0):
    if (topk_ids_out is None and topk_weights_out is None and forced_topk_ids is None
            and router_logits_out is None and not flags and expert_offsets_out is None
            and pair_rows_out is None and not wait_limit_ns):
        return None
    return ctypes.byref(moe_forward_opts_t(
        _ptr(topk_ids_out), _ptr(topk_weights_out), _ptr(forced_topk_ids),
        _ptr(router_logits_out), flags, 0, _ptr(expert_offsets_out), _ptr(pair_rows_out),
        wait_limit_ns))


def moe_forward(h, x, y, T: Optional[int] = None, topk_ids_out=None, topk_weights_out=None,
                forced_topk_ids=None, router_logits_out=None, flags: int = 0, stream=None,
                expert_offsets_out=None, pair_rows_out=None, wait_limit_ns: int = 0):
    """y = MoE(x); x and y are BF16 [T, hidden] device tensors."""
    T = x.shape[0] if T is None else T
    st = _lib.moe_forward(h, _ptr(x), T, _ptr(y),
                          _opts(topk_ids_out, topk_weights_out, forced_topk_ids,
                                router_logits_out, flags, expert_offsets_out, pair_rows_out,
                                wait_limit_ns),
                          _stream(stream))
    _check(st, "moe_forward", h)


def moe_forward_host(h, x_host, y_host, T: Optional[int] = None, flags: int = 0, stream=None):
    """The same from host (CPU, ideally pinned) BF16 tensors; synchronises."""
    T = x_host.shape[0] if T is None else T
    st = _lib.moe_forward_host(h, _ptr(x_host), T, _ptr(y_host),
                               _opts(flags=flags), _stream(stream))
    _check(st, "moe_forward_host", h)


def moe_forward_host_async(h, x_host, y_host, T: Optional[int] = None, flags: int = 0,
                           stream=None):
    """Pipelined host-memory forward (returns at once); keep x_host unchanged and
    y_host unread, and both alive, until moe_host_wait(h) returns."""
    T = x_host.shape[0] if T is None else T
    st = _lib.moe_forward_host_async(h, _ptr(x_host), T, _ptr(y_host),
                                     _opts(flags=flags), _stream(stream))
    _check(st, "moe_forward_host_async", h)


def moe_host_wait(h):
    _check(_lib.moe_host_wait(h), "moe_host_wait", h)


def moe_get_device_status(h) -> int:
    v = ctypes.c_uint32(0)
    _check(_lib.moe_get_device_status(h, ctypes.byref(v)), "moe_get_device_status", h)
    return v.value


def moe_profile_enable(h, max_forwards: int):
    _check(_lib.moe_profile_enable(h, max_forwards), "moe_profile_enable", h)


def moe_profile_read(h, max_forwards: int):
    """List of per-forward lists of MOE_NUM_PHASES phase times in ms."""
    cap = max_forwards * MOE_NUM_PHASES
    buf = (ctypes.c_float * max(cap, 1))()
    n = ctypes.c_int32(0)
    _check(_lib.moe_profile_read(h, buf, cap, ctypes.byref(n)), "moe_profile_read", h)
    n = min(n.value, max_forwards)
    return [[buf[i * MOE_NUM_PHASES + p] for p in range(MOE_NUM_PHASES)] for i in range(n)]


def moe_router_topk_noalloc(x, router_weight, e_score_correction_bias, num_experts_per_tok: int,
                            topk_ids, topk_weights, norm_topk_prob: int = 1,
                            routed_scaling_factor: float = 2.827, T: Optional[int] = None,
                            stream=None):
    """Routing only, with the library's static scratch (no allocation)."""
    T = x.shape[0] if T is None else T
    E, d = router_weight.shape
    st = _lib.moe_router_topk_noalloc(_ptr(x), T, _ptr(router_weight),
                                      _ptr(e_score_correction_bias), d, E, num_experts_per_tok,
                                      norm_topk_prob, routed_scaling_factor, _ptr(topk_ids),
                                      _ptr(topk_weights), _stream(stream))
    _check(st, "moe_router_topk_noalloc")


def moe_act_quant_e4m3(x, q, scales, stream=None):
    """Per-row, per-128-column e4m3 quantisation of a BF16 [rows, cols] tensor."""
    rows, cols = x.shape
    st = _lib.moe_act_quant_e4m3(_ptr(x), rows, cols, _ptr(q), _ptr(scales), _stream(stream))
    _check(st, "moe_act_quant_e4m3")


def moe_combine_rows(pair_out, weights, shared_out, y, stream=None):
    """y[t] = sum_j weights[t, j] * pair_out[t * k + j] + shared_out[t] (BF16
    rows in (token, slot) order; shared_out may be None)."""
    T, k = weights.shape
    st = _lib.moe_combine_rows(_ptr(pair_out), _ptr(weights), _ptr(shared_out), T,
                               pair_out.shape[1], k, _ptr(y), _stream(stream))
    _check(st, "moe_combine_rows")


def moe_launch_count(h) -> int:
    return int(_lib.moe_launch_count(h))


def moe_destroy(h):
    _lib.moe_destroy(h)
