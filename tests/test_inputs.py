"""Checks on the seeded input recipe (CPU only)."""

import json
import math
import os

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import inputs
from oracle import moe_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "zipf_beta.json")


def test_deterministic_and_distinct():
    cfg = inputs.CONFIGS["tiny_fp32"]
    a = inputs.routing_inputs(cfg)
    b = inputs.routing_inputs(cfg)
    for u, v in zip(a, b):
        assert torch.equal(u, v)
    x, w_r, bias = a
    assert x.dtype == torch.float32 and w_r.shape == (16, 128) and bias.shape == (16,)
    assert not torch.equal(x[:16, :16], w_r[:16, :16])
    w1, w3, w2, ws1, ws3, ws2 = inputs.expert_weights(cfg)
    assert not torch.equal(w1, w3)
    assert w2.shape == (16, 128, 64) and ws1.shape == (64, 128) and ws2.shape == (128, 64)


def test_distributions():
    cfg = inputs.CONFIGS["softmax_nogroup"].with_(T=512)
    x, w_r, bias = inputs.routing_inputs(cfg)
    assert bias is None and x.dtype == torch.bfloat16
    assert abs(x.float().std().item() - 1.0) < 0.01
    assert abs(w_r.float().std().item() * math.sqrt(cfg.dim) - 1.0) < 0.02
    cfg2 = inputs.CONFIGS["v3_decode"]
    _, _, b2 = inputs.routing_inputs(cfg2)
    assert abs(b2.std().item() - 0.1) < 0.02          # variance 0.01


def test_router_weight_shape_matches_page_count():
    # page "DeepSeek-V3.2-Exp - Expert scores": 7168 x 256 = 1,835,008 router
    # parameters per MoE block, held [out, in]
    cfg = inputs.CONFIGS["v3_decode"]
    _, w_r, _ = inputs.routing_inputs(cfg.with_(T=1))
    assert tuple(w_r.shape) == (256, 7168) and w_r.numel() == 1_835_008


def test_zipf_beta_matches_calibration():
    with open(GOLD) as f:
        g = json.load(f)
    assert g["beta"] == inputs.ZIPF_BETA and g["zipf_s"] == inputs.ZIPF_S


@pytest.mark.slow
def test_zipf_workload_is_skewed():
    # the skew property the workload is defined by, re-derived with the oracle
    cfg = inputs.CONFIGS["v3_zipf"]
    x, w_r, bias = inputs.routing_inputs(cfg)
    z = O.router_logits(x.float().numpy(), w_r.float().numpy())
    r = O.route(z, bias.numpy().astype(np.float64), n_groups=8, topk_groups=4, topk=8,
                score_func="sigmoid", route_scale=2.5)
    c = O.dispatch(r["idx"], 256)["counts"]
    assert c.max() > 10 * (cfg.T * cfg.topk / 256)
    assert (c == 0).sum() >= 1
    with open(GOLD) as f:
        assert c.tolist() == json.load(f)["counts"]
