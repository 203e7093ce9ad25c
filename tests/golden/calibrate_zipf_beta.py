"""Find the scale beta of the Zipf-skewed selection bias and write it to
tests/golden/zipf_beta.json.

The skewed DeepSeek-V3-shape workload (T=8192, 256 experts, 8 groups, top-4
groups, top-8) draws its bias as beta * (ln p_{pi(e)} - mean) with
p_r ~ r^-1.2 over a seeded permutation pi of the experts. Beta is the
smallest value (to 1e-4, by bisection) for which the oracle's routing of the
workload's x and router weight gives the largest expert more than 10x the mean
token count and leaves at least one expert with no tokens. Router logits are
computed once in float64; each bisection step only re-runs selection.

Run from the repository root:  python tests/golden/calibrate_zipf_beta.py
"""

import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from mixture_experts_layer_42_b200 import inputs  # noqa: E402
from oracle import moe_oracle as O  # noqa: E402


def counts_for(cfg, z, beta):
    bias = inputs.zipf_bias(cfg, beta).numpy().astype(np.float64)
    r = O.route(z, bias, n_groups=cfg.n_groups, topk_groups=cfg.topk_groups, topk=cfg.topk,
                score_func=cfg.score, route_scale=cfg.route_scale)
    return O.dispatch(r["idx"], cfg.n_routed)["counts"]


def skewed(cfg, counts):
    mean = cfg.T * cfg.topk / cfg.n_routed
    return counts.max() > 10 * mean and counts.min() == 0


def main():
    cfg = inputs.CONFIGS["v3_zipf"]
    x, w_r, _ = inputs.routing_inputs(cfg.with_(bias="none"))
    z = O.router_logits(x.float().numpy(), w_r.float().numpy())
    lo, hi = 0.0, 0.05
    while not skewed(cfg, counts_for(cfg, z, hi)):
        lo, hi = hi, hi * 2
        assert hi < 100
    while hi - lo > 1e-4:
        mid = 0.5 * (lo + hi)
        if skewed(cfg, counts_for(cfg, z, mid)):
            hi = mid
        else:
            lo = mid
    beta = round(hi, 4)
    if not skewed(cfg, counts_for(cfg, z, beta)):
        beta = round(hi + 1e-4, 4)
    c = counts_for(cfg, z, beta)
    out = dict(beta=beta, zipf_s=inputs.ZIPF_S, T=cfg.T, topk=cfg.topk, n_routed=cfg.n_routed,
               mean_count=cfg.T * cfg.topk / cfg.n_routed, max_count=int(c.max()),
               zero_experts=int((c == 0).sum()), counts=c.tolist())
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_beta.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps({k: v for k, v in out.items() if k != "counts"}))


if __name__ == "__main__":
    main()
