"""Pins for the oracle's expert math and combine (CPU only): closed forms and
reductions to library routines (torch.nn.functional in float64)."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import moe_oracle as O


def _sig(v):
    return 1.0 / (1.0 + np.exp(-v))


def test_identity_expert_closed_form():
    # I = D, w1 = w3 = Id, w2 = c_e * Id: E_e(x)_d = c_e * x_d^2 * sigmoid(x_d),
    # so y_d = x_d^2 sigmoid(x_d) * sum_j w_j c_{idx_j} (shared MLP zeroed).
    rng = np.random.default_rng(11)
    T, D, E, k = 40, 16, 8, 3
    x = rng.standard_normal((T, D))
    c = 2.0 ** np.arange(E)                       # distinct powers of two
    eye = np.eye(D)
    experts = lambda e: (eye, eye, c[e] * eye)
    zero = np.zeros((D, D))
    z = rng.standard_normal((T, E))
    r = O.route(z, rng.standard_normal(E) * 0.1, n_groups=4, topk_groups=2, topk=k,
                score_func="sigmoid", route_scale=2.5)
    y = O.moe_layer(x, r["weights"], r["idx"], experts, (zero, zero, zero))
    expect = x ** 2 * _sig(x) * (r["weights"] * c[r["idx"]]).sum(-1, keepdims=True)
    np.testing.assert_allclose(y, expect, rtol=1e-13, atol=1e-13)


def test_zero_w1_gives_shared_only():
    rng = np.random.default_rng(12)
    T, D, I, Is, E = 20, 24, 16, 32, 6
    x = rng.standard_normal((T, D))
    z = rng.standard_normal((T, E))
    r = O.route(z, None, n_groups=1, topk_groups=1, topk=2, score_func="softmax", route_scale=1.0)
    experts = lambda e: (np.zeros((I, D)), rng.standard_normal((I, D)), rng.standard_normal((D, I)))
    shared = (rng.standard_normal((Is, D)), rng.standard_normal((Is, D)), rng.standard_normal((D, Is)))
    y = O.moe_layer(x, r["weights"], r["idx"], experts, shared)
    xs = torch.from_numpy(x)
    s = F.linear(F.silu(F.linear(xs, torch.from_numpy(shared[0]))) * F.linear(xs, torch.from_numpy(shared[1])),
                 torch.from_numpy(shared[2])).numpy()
    np.testing.assert_allclose(y, s, rtol=1e-12, atol=1e-12)


def test_single_expert_is_dense_swiglu():
    # E = 1, k = 1, G = 1, sigmoid: the weight is s/s * route_scale, so the layer
    # is route_scale * SwiGLU(x) + shared(x): a dense MLP, checked against
    # torch.nn.functional.linear / silu in float64.
    rng = np.random.default_rng(13)
    T, D, I = 33, 40, 24
    x = rng.standard_normal((T, D))
    w_r = rng.standard_normal((1, D))
    w1, w3, w2 = rng.standard_normal((I, D)), rng.standard_normal((I, D)), rng.standard_normal((D, I))
    ws1, ws3, ws2 = rng.standard_normal((8, D)), rng.standard_normal((8, D)), rng.standard_normal((D, 8))
    out = O.moe_forward(x, w_r, None, lambda e: (w1, w3, w2), (ws1, ws3, ws2), n_groups=1,
                        topk_groups=1, topk=1, score_func="sigmoid", route_scale=1.75)
    assert np.all(out["idx"] == 0)
    np.testing.assert_allclose(out["weights"], 1.75, rtol=1e-15)
    t = lambda a: torch.from_numpy(a)
    mlp = lambda a, b, c: F.linear(F.silu(F.linear(t(x), t(a))) * F.linear(t(x), t(b)), t(c))
    ref = (1.75 * mlp(w1, w3, w2) + mlp(ws1, ws3, ws2)).numpy()
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_layer_matches_library_per_token():
    # every routed term and the shared term recomputed per token with
    # torch.nn.functional in float64 (no rounding), summed with the weights
    rng = np.random.default_rng(14)
    T, D, I, E, k = 15, 32, 16, 12, 3
    x = rng.standard_normal((T, D))
    W = [(rng.standard_normal((I, D)), rng.standard_normal((I, D)), rng.standard_normal((D, I))) for _ in range(E)]
    sh = (rng.standard_normal((I, D)), rng.standard_normal((I, D)), rng.standard_normal((D, I)))
    out = O.moe_forward(x, rng.standard_normal((E, D)), rng.standard_normal(E) * 0.1, lambda e: W[e], sh,
                        n_groups=4, topk_groups=2, topk=k, score_func="sigmoid", route_scale=2.5)
    t = torch.from_numpy
    for tok in range(T):
        xv = t(x[tok:tok + 1])
        acc = torch.zeros(1, D, dtype=torch.float64)
        for j in range(k):
            a, b, c = W[out["idx"][tok, j]]
            acc += out["weights"][tok, j] * F.linear(F.silu(F.linear(xv, t(a))) * F.linear(xv, t(b)), t(c))
        acc += F.linear(F.silu(F.linear(xv, t(sh[0]))) * F.linear(xv, t(sh[1])), t(sh[2]))
        np.testing.assert_allclose(out["y"][tok], acc[0].numpy(), rtol=1e-12, atol=1e-12)


def test_token_subset_equals_full():
    rng = np.random.default_rng(15)
    T, D, I, E = 30, 16, 8, 8
    x = rng.standard_normal((T, D))
    W = [(rng.standard_normal((I, D)), rng.standard_normal((I, D)), rng.standard_normal((D, I))) for _ in range(E)]
    kw = dict(n_groups=2, topk_groups=1, topk=2, score_func="sigmoid", route_scale=1.0)
    wr, bias = rng.standard_normal((E, D)), rng.standard_normal(E)
    full = O.moe_forward(x, wr, bias, lambda e: W[e], None, **kw)
    sub = O.moe_forward(x, wr, bias, lambda e: W[e], None, tokens=[3, 17, 29], **kw)
    np.testing.assert_allclose(sub["y"], full["y"][[3, 17, 29]], rtol=1e-13, atol=1e-13)


def test_act_dtype_rounding_points():
    # with act_dtype="bf16" the layer output is a bf16 value, and h is rounded
    # before w2: choose w2 = Id so the expert output is exactly round(h).
    rng = np.random.default_rng(16)
    D = 8
    x = rng.standard_normal((4, D))
    w1, w3 = rng.standard_normal((D, D)), rng.standard_normal((D, D))
    h = O.silu(x @ w1.T) * (x @ w3.T)
    out = O.swiglu(x, w1, w3, np.eye(D), round_h="bf16", round_out=None)
    ref = torch.from_numpy(h).to(torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    # fp64 -> bf16 directly vs via fp32 only differ on fp32 double-rounding ties
    np.testing.assert_array_equal(out, ref)
