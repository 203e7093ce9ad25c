"""The C ABI library loads, exports every symbol include/moe.h declares, and its
host-side logic (config validation, workspace sizing) behaves; no GPU needed:
every call here returns before touching the device."""

import ctypes
import os
import re

import pytest

from mixture_experts_layer_42_b200 import build as B
from mixture_experts_layer_42_b200 import inputs

HEADER = os.path.join(B.ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def M():
    B.build()
    from mixture_experts_layer_42_b200 import binding
    return binding


def _declared():
    with open(HEADER) as f:
        return re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", f.read(), flags=re.M)


def test_exports_every_declared_symbol(M):
    names = _declared()
    assert len(names) >= 11
    assert sorted(names) == sorted(M.EXPORTS)
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(M):
    for st in (0, -1, -2, -3, -4, -5, -6):
        assert M.status_string(st)
    assert M.status_string(-99) == "unknown status"


def _cfg(**kw):
    base = dict(dim=128, n_routed=16, n_groups=4, topk_groups=2, topk=4, moe_inter=64,
                shared_inter=64, score=0, route_scale=1.0, has_bias=1, dtype=1)
    base.update(kw)
    from mixture_experts_layer_42_b200.binding import moe_config
    return moe_config(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, 0),
    (dict(n_routed=15), -1),                   # E % G != 0
    (dict(topk_groups=5), -1),                 # TG > G
    (dict(topk=9), -1),                        # k > TG * E / G: -inf would be picked
    (dict(n_groups=16, topk_groups=4), -1),    # top-2 group score needs >= 2 per group
    (dict(dim=100), -1),                       # bf16 rows not 16-byte multiples
    (dict(dtype=7), -1),
    (dict(score=3), -1),
    (dict(has_bias=2), -1),
    (dict(route_scale=float("inf")), -1),
    (dict(n_routed=2048, n_groups=8), -2),     # beyond the kernel limits
    (dict(topk=33, n_routed=64, n_groups=1, topk_groups=1), -2),
    (dict(n_routed=48, n_groups=4, topk_groups=2), -2),   # group width 12
    (dict(n_routed=96, n_groups=1, topk_groups=1, has_bias=0), 0),
    (dict(n_routed=256, n_groups=8, topk_groups=4, topk=8, dim=7168, moe_inter=2048,
          shared_inter=2048), 0),
    (dict(dtype=0, dim=20), 0),                # fp32 rows need multiples of 4
])
def test_config_validation(M, kw, status):
    n = ctypes.c_size_t(0)
    st = M.raw_status("moe_workspace_size", ctypes.byref(_cfg(**kw)), 64, ctypes.byref(n))
    assert st == status
    if status == 0:
        assert n.value > 0


def test_bad_sizes_and_pointers(M):
    n = ctypes.c_size_t(0)
    c = ctypes.byref(_cfg())
    assert M.raw_status("moe_workspace_size", c, 0, ctypes.byref(n)) == -1        # T < 1
    assert M.raw_status("moe_workspace_size", c, 1 << 40, ctypes.byref(n)) == -2  # T*k > int32
    assert M.raw_status("moe_workspace_size", c, 8, None) == -1
    # null / misaligned device pointers are rejected before any CUDA call
    assert M.raw_status("moe_gate", c, 8, None, None, None, None, None, None, 0, None) == -1
    p = ctypes.c_void_p(0x1008)
    assert M.raw_status("moe_combine", c, 8, p, p, p, None, p, p, 1 << 20, None) == -1
    assert M.raw_status("moe_workspace_init", None, 0, None) == -1
    assert M.raw_status("moe_check_error", ctypes.c_void_p(0x1001), None) == -1
    assert M.raw_status("moe_select_expert_kernel", 5) == -1
    assert M.raw_status("moe_select_fp8_kernel", 3) == -1
    assert M.raw_status("moe_select_fp8_kernel", -1) == -1
    for which in (M.MOE_FP8_KERNEL_TOKENS_ON_M, M.MOE_FP8_KERNEL_TOKENS_ON_N, M.MOE_FP8_KERNEL_AUTO):
        assert M.raw_status("moe_select_fp8_kernel", which) == 0


def test_fp8_form_for_a_batch(M):
    # AUTO: tokens on M above 16 rows per expert on average (T * k > 16 * E)
    from mixture_experts_layer_42_b200 import inputs
    cfg = inputs.CONFIGS["v3_decode_fp8"]                   # k = 8, E = 256: T = 512 is 16 rows
    assert M.moe_fp8_kernel_for(cfg, 512) == M.MOE_FP8_KERNEL_TOKENS_ON_N
    assert M.moe_fp8_kernel_for(cfg, 513) == M.MOE_FP8_KERNEL_TOKENS_ON_M
    assert M.moe_fp8_kernel_for(cfg, 0) == -1
    try:
        M.moe_select_fp8_kernel(M.MOE_FP8_KERNEL_TOKENS_ON_M)
        assert M.moe_fp8_kernel_for(cfg, 1) == M.MOE_FP8_KERNEL_TOKENS_ON_M
        M.moe_select_fp8_kernel(M.MOE_FP8_KERNEL_TOKENS_ON_N)
        assert M.moe_fp8_kernel_for(cfg, 8192) == M.MOE_FP8_KERNEL_TOKENS_ON_N
    finally:
        M.moe_select_fp8_kernel(M.MOE_FP8_KERNEL_AUTO)


def test_workspace_too_small_is_rejected_before_launch(M):
    n = ctypes.c_size_t(0)
    c = ctypes.byref(_cfg())
    assert M.raw_status("moe_workspace_size", c, 64, ctypes.byref(n)) == 0
    p = ctypes.c_void_p(0x10000)
    st = M.raw_status("moe_combine", c, 64, p, p, p, None, p, p, n.value - 1, None)
    assert st == -3
    st = M.raw_status("moe_combine", c, 64, p, p, p, None, p, None, n.value, None)
    assert st == -3


def test_workspace_size_grows_with_tokens(M):
    for name in ("tiny_fp32", "v3_decode", "softmax_nogroup"):
        cfg = inputs.CONFIGS[name]
        a = M.moe_workspace_size(cfg, 64)
        b = M.moe_workspace_size(cfg, 4096)
        assert b > a > 0
    cfg = inputs.CONFIGS["v3_prefill"]
    ws = M.moe_workspace_size(cfg, cfg.T)
    # y_perm + h dominate (no permuted copy of x): T*k*D*2 + T*k*I*2 bytes
    approx = cfg.T * 8 * 7168 * 2 + cfg.T * 8 * 2048 * 2
    assert approx < ws < approx * 1.2


def test_stall_hook_validates_its_argument(M):
    assert M.raw_status("moe_debug_stall_pipeline", 3) == -1
    assert M.raw_status("moe_debug_stall_pipeline", -1) == -1
    assert M.raw_status("moe_debug_stall_pipeline", 0) == 0


def test_launch_count(M):
    # bf16 on the one-CTA tensor-core kernel: the expert GEMMs follow one
    # kernel that writes their per-expert A maps; a small batch that reads
    # its rows from x is dispatched by one kernel instead of three
    assert M.moe_forward_launch_count(inputs.CONFIGS["v3_decode"], 128) == 7
    assert M.moe_forward_launch_count(inputs.CONFIGS["v3_prefill"], 8192) == 9
    assert M.moe_forward_launch_count(inputs.CONFIGS["tiny_fp32"], 64) == 6
    assert M.moe_forward_launch_count(inputs.CONFIGS["tiny_fp32"], 4096) == 8
    M.moe_select_expert_kernel(M.MOE_EXPERT_KERNEL_TCGEN05_PAIR)
    try:
        assert M.moe_forward_launch_count(inputs.CONFIGS["v3_decode"], 128) == 8
    finally:
        M.moe_select_expert_kernel(M.MOE_EXPERT_KERNEL_AUTO)
    assert M.moe_forward_launch_count(inputs.CONFIGS["v3_decode"], 0) == -1
