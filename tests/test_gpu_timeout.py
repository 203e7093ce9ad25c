"""The failure path of the tensor-core pipeline, on the GPU, without a fault:
a test hook makes one CTA's MMA thread wait on a barrier phase that nothing
completes. The wait runs out after its 1 s limit, the launch drains what it
has in flight and returns, and the host reads MOE_ERR_TIMEOUT from the
workspace's error word. The context stays usable: the next call succeeds and
matches the oracle."""

import time

import pytest
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import inputs
from tests.gpu_util import Layer, forward_parity

pytestmark = pytest.mark.gpu


def _cfg():
    return inputs.MoEConfig("stall", T=300, dim=384, n_routed=16, n_groups=4, topk_groups=2, topk=4,
                            moe_inter=192, n_shared=1, score="sigmoid", bias="normal",
                            route_scale=2.5, dtype="bf16", seed=5)


def test_pipeline_wait_runs_out_and_is_reported():
    cfg = _cfg()
    L = Layer(cfg)
    ws = M.alloc_workspace(cfg, L.T)
    y = torch.empty(L.T, cfg.dim, dtype=cfg.torch_dtype, device="cuda")
    w1, w3, w2, ws1, ws3, ws2 = L.w
    M.moe_debug_stall_pipeline(1)
    try:
        t0 = time.time()
        M.moe_forward(cfg, L.x, L.w_r, L.bias, w1, w3, w2, ws1, ws3, ws2, y, ws)
        status = M.moe_check_error(ws)          # synchronises
        elapsed = time.time() - t0
    finally:
        M.moe_debug_stall_pipeline(0)
    assert status == M.MOE_ERR_TIMEOUT
    assert 0.9 < elapsed < 30
    assert M.moe_check_error(ws) == M.MOE_OK    # read and cleared
    # the same context: the next forward is exact
    err, r, nt = forward_parity(L)
    assert err < 2e-2


@pytest.mark.parametrize("form", ["tokens_on_n", "tokens_on_m"])
def test_fp8_pipeline_wait_runs_out_and_is_reported(form):
    # the same hook on the FP8 up-projection, in each of its two forms
    from tests.test_gpu_fp8 import FORMS, Fp8Layer, _parity, small
    cfg = small(T=300, seed=5)
    F = Fp8Layer(Layer(cfg))
    M.moe_select_fp8_kernel(FORMS[form])
    try:
        L = F.L
        ws = M.alloc_workspace_fp8(cfg, L.T)
        y = torch.empty(L.T, cfg.dim, dtype=torch.bfloat16, device="cuda")
        M.moe_debug_stall_pipeline(1)
        try:
            t0 = time.time()
            M.moe_forward_fp8(cfg, L.x, L.w_r, L.bias, F.fw, y, ws)
            status = M.moe_check_error(ws)      # synchronises
            elapsed = time.time() - t0
        finally:
            M.moe_debug_stall_pipeline(0)
        assert status == M.MOE_ERR_TIMEOUT
        assert 0.9 < elapsed < 30
        assert M.moe_check_error(ws) == M.MOE_OK
        # the same context: the next FP8 forward matches the oracle
        err, *_ = _parity(cfg)
        assert err < 2e-2
    finally:
        M.moe_select_fp8_kernel(M.MOE_FP8_KERNEL_AUTO)
