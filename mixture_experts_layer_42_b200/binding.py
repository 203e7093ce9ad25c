"""Python binding of libmoe.so (the C ABI declared in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels. Tensors are torch CUDA tensors (contiguous); each function passes
their device pointers, the sizes and the caller's CUDA stream through to the
C entry point of the same name, and raises MoEError on a non-OK status.
Importing this module fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# The in-tree build; MOE_LIB_PATH names another build of the same library
# (for example one compiled with different tile constants, to compare them).
LIB_PATH = os.environ.get("MOE_LIB_PATH") or os.path.join(_PKG, "_lib", "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_CHECK = -5
MOE_ERR_TIMEOUT = -6

MOE_DT_F32, MOE_DT_BF16 = 0, 1
MOE_SCORE_SIGMOID, MOE_SCORE_SOFTMAX = 0, 1
MOE_EXPERT_KERNEL_AUTO, MOE_EXPERT_KERNEL_SIMT, MOE_EXPERT_KERNEL_TCGEN05 = 0, 1, 2
MOE_EXPERT_KERNEL_TCGEN05_PAIR = 3
MOE_FP8_KERNEL_AUTO, MOE_FP8_KERNEL_TOKENS_ON_N, MOE_FP8_KERNEL_TOKENS_ON_M = 0, 1, 2
MOE_STALL_NONE, MOE_STALL_EXPERTS_UP, MOE_STALL_ROUTER = 0, 1, 2

# Every symbol include/moe.h declares.
EXPORTS = ("moe_workspace_size", "moe_workspace_init", "moe_gate", "moe_dispatch",
           "moe_experts_grouped", "moe_combine", "moe_forward", "moe_check_error",
           "moe_status_string", "moe_forward_launch_count", "moe_select_expert_kernel",
           "moe_stage_timing_begin", "moe_stage_timing_end", "moe_gate_noalloc",
           "moe_stage_timing_begin_every", "moe_debug_stall_pipeline",
           "moe_gate_noalloc_check_error", "moe_experts_grouped_gather", "moe_forward_ep",
           "moe_cast_output", "moe_quantize_fp8", "moe_workspace_size_fp8", "moe_forward_fp8",
           "moe_select_fp8_kernel", "moe_fp8_kernel_for")

# Kernels of moe_forward, in launch order.
STAGES = ("router_logits", "router_select", "dispatch_rank", "dispatch_scan", "dispatch_pos",
          "experts_up", "experts_down", "combine")


class moe_config(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("n_routed", ctypes.c_int32), ("n_groups", ctypes.c_int32),
                ("topk_groups", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("moe_inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
                ("score", ctypes.c_int32), ("route_scale", ctypes.c_float),
                ("has_bias", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class moe_fp8_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w1", "w3", "w2", "w1_scale", "w3_scale", "w2_scale",
                 "ws1", "ws3", "ws2", "ws1_scale", "ws3_scale", "ws2_scale")]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m mixture_experts_layer_42_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    C = ctypes.POINTER(moe_config)
    sig = {
        "moe_workspace_size": [C, I64, ctypes.POINTER(SZ)],
        "moe_workspace_init": [P, SZ, P],
        "moe_gate": [C, I64, P, P, P, P, P, P, SZ, P],
        "moe_dispatch": [C, I64, P, P, P, P, P, P, P, P, SZ, P],
        "moe_experts_grouped": [C, I64, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_combine": [C, I64, P, P, P, P, P, P, SZ, P],
        "moe_forward": [C, I64, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_check_error": [P, P],
        "moe_status_string": [I32],
        "moe_forward_launch_count": [C, I64],
        "moe_select_expert_kernel": [I32],
        "moe_select_fp8_kernel": [I32],
        "moe_fp8_kernel_for": [C, I64],
        "moe_stage_timing_begin": [I32],
        "moe_stage_timing_begin_every": [I32, I32],
        "moe_debug_stall_pipeline": [I32],
        "moe_stage_timing_end": [ctypes.POINTER(ctypes.c_float), I32],
        "moe_gate_noalloc": [C, I64, P, P, P, P, P, P],
        "moe_gate_noalloc_check_error": [P, P],
        "moe_experts_grouped_gather": [C, I64, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_forward_ep": [C, I64, I32, I32, I32, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_cast_output": [C, I64, P, P, P],
        "moe_quantize_fp8": [C, P, I64, I64, I32, P, P, P],
        "moe_workspace_size_fp8": [C, I64, ctypes.POINTER(SZ)],
        "moe_forward_fp8": [C, I64, P, P, P, ctypes.POINTER(moe_fp8_weights), P, P, P, P, SZ, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = I32
    lib.moe_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def status_string(status: int) -> str:
    return _lib.moe_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoEError(status, where)


def make_config(cfg) -> moe_config:
    """C config from any object with the fields of inputs.MoEConfig."""
    return moe_config(dim=cfg.dim, n_routed=cfg.n_routed, n_groups=cfg.n_groups,
                      topk_groups=cfg.topk_groups, topk=cfg.topk, moe_inter=cfg.moe_inter,
                      shared_inter=cfg.n_shared * cfg.moe_inter,
                      score=MOE_SCORE_SIGMOID if cfg.score == "sigmoid" else MOE_SCORE_SOFTMAX,
                      route_scale=float(cfg.route_scale), has_bias=1 if cfg.bias != "none" else 0,
                      dtype=MOE_DT_F32 if cfg.dtype == "f32" else MOE_DT_BF16)


def _c(cfg):
    return ctypes.byref(cfg if isinstance(cfg, moe_config) else make_config(cfg))


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream))


def moe_workspace_size(cfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_workspace_size(_c(cfg), int(T), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(_lib.moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _s(stream)),
           "moe_workspace_init")


def alloc_workspace(cfg, T: int, device="cuda") -> torch.Tensor:
    """A zero-initialised workspace for T tokens (torch allocates it)."""
    ws = torch.empty(moe_workspace_size(cfg, T), dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


def moe_gate(cfg, x, w_router, bias, weights, idx, ws, stream=None) -> None:
    _check(_lib.moe_gate(_c(cfg), x.shape[0], _p(x), _p(w_router), _p(bias), _p(weights), _p(idx),
                         _p(ws), ws.numel(), _s(stream)), "moe_gate")


def moe_gate_noalloc(cfg, x, w_router, bias, weights, idx, stream=None) -> None:
    """moe_gate with the library's built-in scratch instead of a workspace."""
    _check(_lib.moe_gate_noalloc(_c(cfg), x.shape[0], _p(x), _p(w_router), _p(bias), _p(weights),
                                 _p(idx), _s(stream)), "moe_gate_noalloc")


def moe_gate_noalloc_check_error(x, stream=None) -> int:
    """Synchronise, read and clear moe_gate_noalloc's built-in error word on
    x's device; returns the status."""
    return int(_lib.moe_gate_noalloc_check_error(_p(x), _s(stream)))


def moe_dispatch(cfg, idx, x, counts, offsets, src, pos, x_perm, ws, stream=None) -> None:
    """x_perm may be None (x is then not read; only the indices are written)."""
    _check(_lib.moe_dispatch(_c(cfg), idx.shape[0], _p(idx), _p(x), _p(counts), _p(offsets), _p(src),
                             _p(pos), _p(x_perm), _p(ws), ws.numel(), _s(stream)), "moe_dispatch")


def moe_experts_grouped(cfg, T, x_perm, offsets, w1, w3, w2, x, ws1, ws3, ws2, y_perm, s, ws,
                        stream=None) -> None:
    _check(_lib.moe_experts_grouped(_c(cfg), int(T), _p(x_perm), _p(offsets), _p(w1), _p(w3), _p(w2),
                                    _p(x), _p(ws1), _p(ws3), _p(ws2), _p(y_perm), _p(s), _p(ws),
                                    ws.numel(), _s(stream)), "moe_experts_grouped")


def moe_experts_grouped_gather(cfg, x, src, offsets, w1, w3, w2, ws1, ws3, ws2, y_perm, s, ws,
                               stream=None) -> None:
    _check(_lib.moe_experts_grouped_gather(_c(cfg), x.shape[0], _p(x), _p(src), _p(offsets), _p(w1),
                                           _p(w3), _p(w2), _p(ws1), _p(ws3), _p(ws2), _p(y_perm), _p(s),
                                           _p(ws), ws.numel(), _s(stream)), "moe_experts_grouped_gather")


def moe_combine(cfg, y_perm, pos, weights, s, y, ws, stream=None) -> None:
    _check(_lib.moe_combine(_c(cfg), y.shape[0], _p(y_perm), _p(pos), _p(weights), _p(s), _p(y),
                            _p(ws), ws.numel(), _s(stream)), "moe_combine")


def moe_forward(cfg, x, w_router, bias, w1, w3, w2, ws1, ws3, ws2, y, ws, weights_out=None,
                idx_out=None, stream=None) -> None:
    _check(_lib.moe_forward(_c(cfg), x.shape[0], _p(x), _p(w_router), _p(bias), _p(w1), _p(w3),
                            _p(w2), _p(ws1), _p(ws3), _p(ws2), _p(y), _p(weights_out), _p(idx_out),
                            _p(ws), ws.numel(), _s(stream)), "moe_forward")


def moe_forward_ep(cfg, expert_begin, expert_end, shared_local, x, w_router, bias, w1, w3, w2,
                   ws1, ws3, ws2, y_partial, ws, weights_out=None, idx_out=None, stream=None) -> None:
    _check(_lib.moe_forward_ep(_c(cfg), x.shape[0], int(expert_begin), int(expert_end),
                               int(shared_local), _p(x), _p(w_router), _p(bias), _p(w1), _p(w3),
                               _p(w2), _p(ws1), _p(ws3), _p(ws2), _p(y_partial), _p(weights_out),
                               _p(idx_out), _p(ws), ws.numel(), _s(stream)), "moe_forward_ep")


def moe_cast_output(cfg, y_sum, y, stream=None) -> None:
    _check(_lib.moe_cast_output(_c(cfg), y.shape[0], _p(y_sum), _p(y), _s(stream)), "moe_cast_output")


def moe_quantize_fp8(cfg, a, block_rows, q, scales, stream=None) -> None:
    """a [rows, cols] (act dtype) -> q [rows, cols] e4m3 (uint8) and scales
    [ceil(rows / block_rows), cols / 128] fp32."""
    a2 = a.reshape(-1, a.shape[-1])
    _check(_lib.moe_quantize_fp8(_c(cfg), _p(a2), a2.shape[0], a2.shape[1], int(block_rows), _p(q),
                                 _p(scales), _s(stream)), "moe_quantize_fp8")


def moe_workspace_size_fp8(cfg, T: int) -> int:
    n = ctypes.c_size_t(0)
    _check(_lib.moe_workspace_size_fp8(_c(cfg), int(T), ctypes.byref(n)), "moe_workspace_size_fp8")
    return n.value


def alloc_workspace_fp8(cfg, T: int, device="cuda") -> torch.Tensor:
    ws = torch.empty(moe_workspace_size_fp8(cfg, T), dtype=torch.uint8, device=device)
    moe_workspace_init(ws)
    return ws


def fp8_weights(w1, w3, w2, s1, s3, s2, ws1=None, ws3=None, ws2=None, ss1=None, ss3=None,
                ss2=None) -> moe_fp8_weights:
    """The C struct of FP8 expert weights from device tensors (kept alive by
    the caller)."""
    return moe_fp8_weights(*[None if t is None else _p(t) for t in
                             (w1, w3, w2, s1, s3, s2, ws1, ws3, ws2, ss1, ss3, ss2)])


def moe_forward_fp8(cfg, x, w_router, bias, fw: moe_fp8_weights, y, ws, weights_out=None,
                    idx_out=None, stream=None) -> None:
    _check(_lib.moe_forward_fp8(_c(cfg), x.shape[0], _p(x), _p(w_router), _p(bias), ctypes.byref(fw),
                                _p(y), _p(weights_out), _p(idx_out), _p(ws), ws.numel(), _s(stream)),
           "moe_forward_fp8")


def moe_check_error(ws, stream=None) -> int:
    """Synchronise, read and clear the device error word; returns the status."""
    return int(_lib.moe_check_error(_p(ws), _s(stream)))


def moe_forward_launch_count(cfg, T: int) -> int:
    return int(_lib.moe_forward_launch_count(_c(cfg), int(T)))


def moe_debug_stall_pipeline(enable: int) -> None:
    _check(_lib.moe_debug_stall_pipeline(int(enable)), "moe_debug_stall_pipeline")


def moe_select_expert_kernel(which: int) -> None:
    _check(_lib.moe_select_expert_kernel(int(which)), "moe_select_expert_kernel")


def moe_select_fp8_kernel(which: int) -> None:
    _check(_lib.moe_select_fp8_kernel(int(which)), "moe_select_fp8_kernel")


def moe_fp8_kernel_for(cfg, T: int) -> int:
    """The FP8 GEMM form moe_forward_fp8 runs for T tokens (MOE_FP8_KERNEL_TOKENS_ON_N / _ON_M)."""
    return int(_lib.moe_fp8_kernel_for(_c(cfg), int(T)))


def moe_stage_timing_begin(max_calls: int) -> None:
    _check(_lib.moe_stage_timing_begin(int(max_calls)), "moe_stage_timing_begin")


def moe_stage_timing_begin_every(max_calls: int, every: int) -> None:
    _check(_lib.moe_stage_timing_begin_every(int(max_calls), int(every)),
           "moe_stage_timing_begin_every")


def moe_stage_timing_end() -> tuple:
    """(calls recorded, {kernel name: total ms over those calls})."""
    ms = (ctypes.c_float * len(STAGES))()
    n = int(_lib.moe_stage_timing_end(ms, len(STAGES)))
    if n < 0:
        raise MoEError(n, "moe_stage_timing_end")
    return n, {name: float(ms[i]) for i, name in enumerate(STAGES)}


def raw_status(name: str, *args) -> int:
    """Call a C entry point with raw ctypes arguments and return its status
    (for tests of the argument checks)."""
    return int(getattr(_lib, name)(*args))
