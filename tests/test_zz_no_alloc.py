"""moe_gate_noalloc: the router entry point for callers that cannot allocate
device memory (a plugin in a host framework that owns every byte of device
memory through its own pool, a serving loop where cudaMalloc is off limits
because it can synchronise the device). It keeps its scratch, and its error
word, in storage built into the library instead of a caller workspace.

Checked through the C ABI on several calls in a row, with the tolerance of the
other routing tests, against the oracle (indices equal on every token whose
oracle margin is at least 1e-6, weights within 1e-6 * route_scale) and against
moe_gate (the workspace entry point). The built-in array keeps the previous
call's partial sums, so back-to-back calls of different shapes also check
that nothing stale is read. A router wait that runs out (a test hook, no
fault) must be reported through the built-in error word and leave the outputs
unwritten. This file is collected last on purpose."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import inputs
from tests.gpu_util import Layer, check_routing

pytestmark = pytest.mark.gpu


def _sentinels(T, k):
    return (torch.full((T, k), -1.0, dtype=torch.float32, device="cuda"),
            torch.full((T, k), -1, dtype=torch.int32, device="cuda"))


def _gate_both(cfg):
    L = Layer(cfg, weights=(None,) * 6)
    T, k = L.T, cfg.topk
    w_ref = torch.empty(T, k, dtype=torch.float32, device="cuda")
    i_ref = torch.empty(T, k, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg, T)
    M.moe_gate(cfg, L.x, L.w_r, L.bias, w_ref, i_ref, ws)
    w_na, i_na = _sentinels(T, k)
    M.moe_gate_noalloc(cfg, L.x, L.w_r, L.bias, w_na, i_na)
    assert M.moe_gate_noalloc_check_error(L.x) == M.MOE_OK
    return L, (w_ref, i_ref), (w_na, i_na)


def _agree(cfg, L, ref, got):
    r = L.oracle_route()
    check_routing(cfg, got[1], got[0], r)                  # against the oracle
    (w_ref, i_ref), (w_na, i_na) = [(w.cpu().numpy(), i.cpu().numpy()) for w, i in (ref, got)]
    same = (i_ref == i_na).all(axis=1)                     # against moe_gate
    assert same[r["margin"] >= 1e-6].all(), "indices differ on a token with margin >= 1e-6"
    assert np.abs(w_ref[same] - w_na[same]).max() <= 1e-6 * cfg.route_scale


def test_noalloc_gate_matches_oracle_and_workspace_gate_on_consecutive_calls():
    calls = [
        inputs.CONFIGS["v3_decode"],                       # 128 x 256: same split count as moe_gate
        inputs.CONFIGS["softmax_nogroup"].with_(T=2048),   # fewer splits fit: different shape, sums
        inputs.CONFIGS["tiny_fp32"],                       # fp32 inputs
        inputs.CONFIGS["v3_decode"].with_(T=4096),         # the largest V3 batch that fits
        inputs.CONFIGS["v3_decode"],                       # back to the first shape
    ]
    for cfg in calls:
        L, ref, got = _gate_both(cfg)
        _agree(cfg, L, ref, got)


def test_noalloc_gate_rejects_shapes_beyond_its_scratch():
    cfg = inputs.CONFIGS["v3_decode"].with_(T=4097)        # 4097 * 256 > 1,048,576 floats
    x = torch.zeros(cfg.T, cfg.dim, dtype=torch.bfloat16, device="cuda")
    w_r = torch.zeros(cfg.n_routed, cfg.dim, dtype=torch.bfloat16, device="cuda")
    bias = torch.zeros(cfg.n_routed, dtype=torch.float32, device="cuda")
    w, i = _sentinels(cfg.T, cfg.topk)
    with pytest.raises(M.MoEError) as e:
        M.moe_gate_noalloc(cfg, x, w_r, bias, w, i)
    assert e.value.status == M.MOE_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert (i == -1).all() and (w == -1.0).all()          # nothing launched


def test_noalloc_gate_reports_a_router_wait_that_ran_out():
    cfg = inputs.CONFIGS["v3_decode"]
    L = Layer(cfg, weights=(None,) * 6)
    w, i = _sentinels(L.T, cfg.topk)
    M.moe_debug_stall_pipeline(M.MOE_STALL_ROUTER)
    try:
        M.moe_gate_noalloc(cfg, L.x, L.w_r, L.bias, w, i)
        torch.cuda.synchronize()
    finally:
        M.moe_debug_stall_pipeline(M.MOE_STALL_NONE)
    # the error stays set until it is read, and holds back later calls' output
    M.moe_gate_noalloc(cfg, L.x, L.w_r, L.bias, w, i)
    torch.cuda.synchronize()
    assert (i == -1).all() and (w == -1.0).all(), "routing written from stale partial sums"
    assert M.moe_gate_noalloc_check_error(L.x) == M.MOE_ERR_TIMEOUT
    assert M.moe_gate_noalloc_check_error(L.x) == M.MOE_OK  # read and cleared
    # the same context: the next call is exact
    M.moe_gate_noalloc(cfg, L.x, L.w_r, L.bias, w, i)
    assert M.moe_gate_noalloc_check_error(L.x) == M.MOE_OK
    check_routing(cfg, i, w, L.oracle_route())
