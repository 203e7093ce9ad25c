"""Seeded synthetic inputs for the MoE layer, shared by the CUDA path and the oracle.

This module only draws numbers: it holds none of the layer's arithmetic (no
routing, no expert math). Both sides of a parity check take their inputs from
here, so they see identical bits.

Distributions (the workloads of the layer):
  * x ~ N(0, 1), drawn in fp32 and rounded to nearest-even into the activation
    dtype (bf16 or fp32).
  * every weight matrix ~ N(0, 1/fan_in): std = 1/sqrt(fan_in), where fan_in is
    the input width of that linear (dim for the router, w1 and w3; the inner
    width for w2). Stored in the activation dtype, layout [out, in] as the
    router weight is on page "DeepSeek-V3.2-Exp - Expert scores".
  * the selection bias, fp32: N(0, 0.01) read as variance 0.01 (std 0.1), or a
    Zipf-shaped bias (below), or absent.

Determinism: every tensor comes from its own torch.Generator, seeded by a hash
of (seed, tensor name, shape). The routing-side tensors (x, router weight,
bias) are always drawn on the CPU, so routing inputs are identical on every
machine; the expert weights may be drawn on the GPU (they are ~22 GB at the
DeepSeek-V3 shape) and are then copied to the host where the oracle needs them.
"""

from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    """One MoE layer shape. Field names follow the Gate/MoE constructor
    arguments on the pages (dim, n_routed_experts, n_expert_groups,
    n_limited_groups, n_activated_experts, moe_inter_dim, n_shared_experts,
    score_func, route_scale)."""

    name: str
    T: int                 # tokens (batch x sequence, flattened)
    dim: int               # model width D
    n_routed: int          # routed experts E
    n_groups: int          # expert groups G (1 = no group limit)
    topk_groups: int       # groups kept per token
    topk: int              # experts per token k
    moe_inter: int         # routed expert inner width I
    n_shared: int          # shared experts S_n; one MLP of width S_n * I
    score: str             # "sigmoid" | "softmax"
    bias: str              # "normal" | "zipf" | "none"
    route_scale: float
    dtype: str             # "f32" | "bf16"
    seed: int = 0
    fp8: bool = False      # expert weights in the FP8 block-scaled layout (quantized from
                           # the drawn bf16 weights by the library)

    @property
    def shared_inter(self) -> int:
        return self.n_shared * self.moe_inter

    @property
    def has_bias(self) -> bool:
        return self.bias != "none"

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)


# The five workloads of the layer.
CONFIGS = {
    # Tiny fp32 layer: 16 experts in 4 groups, 2 groups kept, top-4.
    "tiny_fp32": MoEConfig("tiny_fp32", T=64, dim=128, n_routed=16, n_groups=4,
                           topk_groups=2, topk=4, moe_inter=64, n_shared=1,
                           score="sigmoid", bias="normal", route_scale=1.0, dtype="f32"),
    # DeepSeek-V3 shape, decode batch of 128 tokens.
    "v3_decode": MoEConfig("v3_decode", T=128, dim=7168, n_routed=256, n_groups=8,
                           topk_groups=4, topk=8, moe_inter=2048, n_shared=1,
                           score="sigmoid", bias="normal", route_scale=2.5, dtype="bf16"),
    # DeepSeek-V3 shape, prefill of 8192 tokens.
    "v3_prefill": MoEConfig("v3_prefill", T=8192, dim=7168, n_routed=256, n_groups=8,
                            topk_groups=4, topk=8, moe_inter=2048, n_shared=1,
                            score="sigmoid", bias="normal", route_scale=2.5, dtype="bf16"),
    # Softmax routing, no bias, no groups, no renormalisation.
    "softmax_nogroup": MoEConfig("softmax_nogroup", T=4096, dim=2048, n_routed=64, n_groups=1,
                                 topk_groups=1, topk=6, moe_inter=1408, n_shared=2,
                                 score="softmax", bias="none", route_scale=1.0, dtype="bf16"),
    # DeepSeek-V3 prefill with a Zipf(1.2)-skewed expert popularity.
    "v3_zipf": MoEConfig("v3_zipf", T=8192, dim=7168, n_routed=256, n_groups=8,
                         topk_groups=4, topk=8, moe_inter=2048, n_shared=1,
                         score="sigmoid", bias="zipf", route_scale=2.5, dtype="bf16"),
    # The decode batch with its expert weights in the FP8 block-scaled layout.
    "v3_decode_fp8": MoEConfig("v3_decode_fp8", T=128, dim=7168, n_routed=256, n_groups=8,
                               topk_groups=4, topk=8, moe_inter=2048, n_shared=1,
                               score="sigmoid", bias="normal", route_scale=2.5, dtype="bf16",
                               fp8=True),
    # The prefill batch with its expert weights in the FP8 block-scaled layout.
    "v3_prefill_fp8": MoEConfig("v3_prefill_fp8", T=8192, dim=7168, n_routed=256, n_groups=8,
                                topk_groups=4, topk=8, moe_inter=2048, n_shared=1,
                                score="sigmoid", bias="normal", route_scale=2.5, dtype="bf16",
                                fp8=True),
}

# Zipf exponent of the skewed workload and the scale beta of its bias. Beta was
# found by bisection with the oracle's router on this module's x and router
# weight for "v3_zipf" (tests/golden/calibrate_zipf_beta.py writes
# tests/golden/zipf_beta.json; a CPU test checks that the resulting counts show
# the skew: the largest expert gets > 10x the mean and some expert gets none).
ZIPF_S = 1.2
ZIPF_BETA = 0.0771


def _stream_seed(seed: int, name: str, shape) -> int:
    key = f"{seed}|{name}|{'x'.join(str(int(s)) for s in shape)}".encode()
    return int.from_bytes(hashlib.sha256(key).digest()[:8], "little") & ((1 << 63) - 1)


def _normal(name: str, shape, std: float, seed: int, device, out_dtype) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(_stream_seed(seed, name, shape))
    t = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(out_dtype)


def zipf_bias(cfg: MoEConfig, beta: float) -> torch.Tensor:
    """Selection bias whose ordering follows Zipf(s) over a seeded permutation
    of the experts: bias_e = beta * (ln p_{pi(e)} - mean), p_r ~ r^-s."""
    E = cfg.n_routed
    g = torch.Generator(device="cpu")
    g.manual_seed(_stream_seed(cfg.seed, "zipf_perm", (E,)))
    perm = torch.randperm(E, generator=g)
    ranks = torch.arange(1, E + 1, dtype=torch.float64)
    logp = -ZIPF_S * torch.log(ranks)
    logp = logp - torch.logsumexp(logp, 0)
    lp = logp[perm]
    return (beta * (lp - lp.mean())).to(torch.float32)


def routing_inputs(cfg: MoEConfig, T: Optional[int] = None):
    """x [T, dim], router weight [E, dim] (activation dtype) and the bias
    [E] fp32 (or None); always drawn on the CPU."""
    T = cfg.T if T is None else T
    dt = cfg.torch_dtype
    x = _normal("x", (T, cfg.dim), 1.0, cfg.seed, "cpu", dt)
    w_router = _normal("w_router", (cfg.n_routed, cfg.dim), 1.0 / math.sqrt(cfg.dim), cfg.seed, "cpu", dt)
    if cfg.bias == "normal":
        bias = _normal("bias", (cfg.n_routed,), 0.1, cfg.seed, "cpu", torch.float32)
    elif cfg.bias == "zipf":
        bias = zipf_bias(cfg, ZIPF_BETA)
    else:
        bias = None
    return x, w_router, bias


def expert_weights(cfg: MoEConfig, device="cpu"):
    """Routed expert weights w1, w3 [E, I, D] and w2 [E, D, I] plus the shared
    MLP ws1, ws3 [I_s, D] and ws2 [D, I_s], all [out, in], drawn on `device`
    one expert at a time (each expert has its own stream)."""
    E, D, I, Is = cfg.n_routed, cfg.dim, cfg.moe_inter, cfg.shared_inter
    dt = cfg.torch_dtype
    sd, si = 1.0 / math.sqrt(D), 1.0 / math.sqrt(I)
    w1 = torch.empty(E, I, D, dtype=dt, device=device)
    w3 = torch.empty(E, I, D, dtype=dt, device=device)
    w2 = torch.empty(E, D, I, dtype=dt, device=device)
    for e in range(E):
        w1[e] = _normal(f"w1.{e}", (I, D), sd, cfg.seed, device, dt)
        w3[e] = _normal(f"w3.{e}", (I, D), sd, cfg.seed, device, dt)
        w2[e] = _normal(f"w2.{e}", (D, I), si, cfg.seed, device, dt)
    if Is > 0:
        ws1 = _normal("ws1", (Is, D), sd, cfg.seed, device, dt)
        ws3 = _normal("ws3", (Is, D), sd, cfg.seed, device, dt)
        ws2 = _normal("ws2", (D, Is), 1.0 / math.sqrt(Is), cfg.seed, device, dt)
    else:
        ws1 = ws3 = ws2 = None
    return w1, w3, w2, ws1, ws3, ws2


def small_config(**kw) -> MoEConfig:
    """A small layer for edge cases; defaults mirror the tiny config."""
    base = CONFIGS["tiny_fp32"].with_(name="small")
    return base.with_(**kw)
