"""The expert-parallel layer's share kernel (moe_forward_ep) and final cast
(moe_cast_output) on one GPU, through the C ABI. The ranks of an N-way
partition run one after another on the same GPU (nothing waits on another
rank: each share is an independent forward), their fp32 shares are summed on
the device in rank order -- the all_reduce's sum -- and cast once. The result
is compared with the oracle's expert-parallel layer (each rank rounds its own
slice of the shared MLP) and with the one-GPU moe_forward; with one rank it
is moe_forward bit for bit."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import ep, inputs
from oracle import moe_oracle as O
from tests.gpu_util import Layer, check_routing, check_y, host, to_np

pytestmark = pytest.mark.gpu


def bf16_small(**kw):
    base = inputs.MoEConfig("ep_small", T=300, dim=384, n_routed=16, n_groups=4, topk_groups=2,
                            topk=4, moe_inter=192, n_shared=1, score="sigmoid", bias="normal",
                            route_scale=2.5, dtype="bf16", seed=9)
    return base.with_(**kw)


def _ep_forward(L, world):
    cfg = L.cfg
    total = torch.zeros(L.T, cfg.dim, dtype=torch.float32, device="cuda")
    idxs = []
    for r in range(world):
        rank = ep.EPLayer(cfg, L.T, L.w, world, r, "cuda")
        idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
        total += rank.partial(L.x, L.w_r, L.bias, idx_out=idx)
        assert M.moe_check_error(rank.ws) == M.MOE_OK
        idxs.append(idx)
    y = torch.empty(L.T, cfg.dim, dtype=cfg.torch_dtype, device="cuda")
    M.moe_cast_output(cfg, total, y)
    torch.cuda.synchronize()
    return y, idxs


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("cfg", [
    bf16_small(),
    bf16_small(T=77, n_routed=64, n_groups=8, topk_groups=3, topk=6, n_shared=2),
    bf16_small(score="softmax", bias="none", n_groups=1, topk_groups=1, n_shared=0),
    inputs.CONFIGS["tiny_fp32"],
], ids=["bf16", "bf16_64e_shared2", "softmax_no_shared", "tiny_fp32"])
def test_ep_shares_sum_to_the_layer(cfg, world):
    L = Layer(cfg)
    y1, w1_, idx1 = L.forward()                       # the one-GPU layer
    y, idxs = _ep_forward(L, world)
    for i in idxs:                                     # every rank routes alike
        assert torch.equal(i, idx1)
    if world == 1:
        assert torch.equal(y, y1)
        return
    r = L.oracle_route()
    differs = check_routing(cfg, idx1, w1_, r)
    rows = np.nonzero(~differs)[0]
    yref = O.moe_layer_ep(host(L.x), r["weights"], r["idx"], L.experts_np(), L.shared_np(),
                          n_experts=cfg.n_routed, world_size=world, act_dtype=cfg.dtype, tokens=rows)
    err = check_y(cfg, to_np(y)[rows], yref)
    assert err < (1e-4 if cfg.dtype == "f32" else 2e-2)
    check_y(cfg, to_np(y), to_np(y1))                 # and the one-GPU layer


def test_ep_v3_decode_eight_ranks():
    # the DeepSeek-V3 decode batch split over eight ranks: 32 experts and a
    # 256-wide shared slice each
    cfg = inputs.CONFIGS["v3_decode"]
    L = Layer(cfg)
    y1, _, idx1 = L.forward()
    y, idxs = _ep_forward(L, 8)
    assert all(torch.equal(i, idx1) for i in idxs)
    check_y(cfg, to_np(y), to_np(y1))


def test_ep_argument_checks():
    cfg = bf16_small(T=8)
    L = Layer(cfg)
    y32 = torch.empty(L.T, cfg.dim, dtype=torch.float32, device="cuda")
    ws = M.alloc_workspace(cfg, L.T)
    w1, w3, w2, ws1, ws3, ws2 = L.w
    for b, e, sl in [(4, 4, 0), (-1, 4, 0), (0, 17, 0), (0, 4, 200), (0, 4, 4)]:
        with pytest.raises(M.MoEError) as ex:
            M.moe_forward_ep(cfg, b, e, sl, L.x, L.w_r, L.bias, w1, w3, w2, ws1, ws3, ws2, y32, ws)
        assert ex.value.status == M.MOE_ERR_INVALID_ARG
