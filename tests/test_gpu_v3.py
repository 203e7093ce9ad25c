"""GPU parity of the whole layer at the DeepSeek-V3 shape (D=7168, 256
experts in 8 groups, top-4 groups, top-8, I=2048, one shared expert), in the
launch configuration the benchmark times, for the decode batch (T=128, every
token), the prefill batch (T=8192), the Zipf-skewed prefill batch and a batch
of 40000 tokens whose permuted activations pass 2^31 elements.

Routing is checked on every token of every batch. Outputs are checked on every
decode token and on a seeded sample of prefill tokens, 1024 of each 8192-token
batch (which always includes tokens routed to the most and least loaded
experts): a token's output depends
only on its own row, so sampled rows are exact checks of those rows. The three
batches share their expert weights, so one oracle pass over the experts
serves all of them."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import inputs
from oracle import moe_oracle as O
from tests.gpu_util import Layer, check_routing, check_y, host, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

NAMES = ("v3_decode", "v3_prefill", "v3_zipf", "v3_large")
# seeded token sample of the prefill-sized batches: 1024 tokens of the two
# 8192-token workloads, 96 of the 40000-token batch
SAMPLE = {"v3_prefill": 1024, "v3_zipf": 1024, "v3_large": 96}
# The largest batch: T*k*D = 2.29e9 elements in x_perm and y_perm, past 2^31,
# so rows beyond that point exercise the kernels' 64-bit addressing.
LARGE_T = 40000
ROWS_2_31 = (1 << 31) // 7168 + 1   # first x_perm row past 2^31 elements at D=7168


def config(name):
    if name == "v3_large":
        return inputs.CONFIGS["v3_prefill"].with_(name="v3_large", T=LARGE_T)
    return inputs.CONFIGS[name]


@pytest.fixture(scope="module")
def v3():
    cfg0 = inputs.CONFIGS["v3_decode"]
    weights = inputs.expert_weights(cfg0, "cuda")
    runs = {}
    for name in NAMES:
        cfg = config(name)
        L = Layer(cfg, weights=weights)
        y, wts, idx = L.forward()
        r = L.oracle_route()
        differs = check_routing(cfg, idx, wts, r)
        if differs.any():
            oi = torch.from_numpy(r["idx"].astype(np.int32)).cuda()
            ow = torch.from_numpy(r["weights"].astype(np.float32)).cuda()
            y, _ = L.split(oi, ow)
        if L.T <= 128:
            tokens = np.arange(L.T)
        else:
            rng = np.random.default_rng(7)
            counts = np.bincount(r["idx"].ravel(), minlength=cfg.n_routed)
            hot, cold = int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
            picks = [np.nonzero((r["idx"] == hot).any(1))[0][:4], np.nonzero((r["idx"] == cold).any(1))[0][:4],
                     [0, L.T - 1], rng.choice(L.T, SAMPLE[name], replace=False)]
            if L.T * cfg.topk * cfg.dim > (1 << 31):
                # tokens with a dispatched row past 2^31 elements of x_perm / y_perm
                pos = O.dispatch(r["idx"], cfg.n_routed)["pos"].reshape(L.T, cfg.topk)
                far = np.nonzero((pos >= ROWS_2_31).any(1))[0]
                assert len(far) > 0
                picks.append(rng.choice(far, min(32, len(far)), replace=False))
            tokens = np.unique(np.concatenate(picks))
        runs[name] = dict(L=L, y=to_np(y)[tokens], r=r, tokens=tokens, differs=int(differs.sum()))
        del y
    # one oracle pass over the experts for the rows of all three batches
    xs = np.concatenate([host(runs[n]["L"].x)[runs[n]["tokens"]] for n in NAMES])
    ws = np.concatenate([runs[n]["r"]["weights"][runs[n]["tokens"]] for n in NAMES])
    ids = np.concatenate([runs[n]["r"]["idx"][runs[n]["tokens"]] for n in NAMES])
    L0 = runs[NAMES[0]]["L"]
    yref = O.moe_layer(xs, ws, ids, L0.experts_np(), L0.shared_np(), act_dtype="bf16")
    o = 0
    for n in NAMES:
        k = len(runs[n]["tokens"])
        runs[n]["yref"] = yref[o:o + k]
        o += k
    return runs


@pytest.mark.parametrize("name", NAMES)
def test_v3_layer_parity(v3, name):
    run = v3[name]
    err = check_y(config(name), run["y"], run["yref"])
    assert err < 2e-2
    # only near-ties (oracle margin < 1e-6) may differ; a handful per batch
    assert run["differs"] <= max(2, run["L"].T // 5000)


def test_zipf_batch_is_skewed(v3):
    r = v3["v3_zipf"]["r"]
    counts = np.bincount(r["idx"].ravel(), minlength=256)
    assert counts.max() > 10 * counts.mean() and (counts == 0).any()
