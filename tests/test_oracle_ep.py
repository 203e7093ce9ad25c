"""Pins for the oracle's expert-parallel partition (CPU only): the expert
blocks and shared slices of the MoE class (hackaday page) and
DeepseekV3MoE.__init__ (thataiguy page) cover every expert and inner feature
once, and the ranks' partial outputs add up to the whole layer -- a property
of the layer's math (each expert and each inner feature of the shared MLP
contributes independently), checked against the oracle's own single-rank
layer and against torch's SwiGLU."""

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


@pytest.mark.parametrize("E,N", [(16, 1), (16, 2), (16, 4), (64, 8), (256, 8)])
def test_expert_blocks_cover_every_expert_once(E, N):
    blocks = [O.expert_block(E, N, r) for r in range(N)]
    assert [e for b in blocks for e in b] == list(range(E))
    assert all(len(b) == E // N for b in blocks)
    assert blocks[0].start == 0 and blocks[-1].stop == E


def test_expert_blocks_need_an_even_split():
    with pytest.raises(ValueError):
        O.expert_block(10, 4, 0)


def _small_layer(seed=0, T=40, D=32, I=16, E=16, k=4, Is=32):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, D))
    idx = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    w = rng.uniform(0.1, 1.0, (T, k))
    ex = {e: (rng.standard_normal((I, D)) / np.sqrt(D), rng.standard_normal((I, D)) / np.sqrt(D),
              rng.standard_normal((D, I)) / np.sqrt(I)) for e in range(E)}
    sh = (rng.standard_normal((Is, D)) / np.sqrt(D), rng.standard_normal((Is, D)) / np.sqrt(D),
          rng.standard_normal((D, Is)) / np.sqrt(Is))
    return x, w, idx, ex, sh


@pytest.mark.parametrize("N", [1, 2, 4, 8])
def test_partials_add_up_to_the_layer(N):
    x, w, idx, ex, sh = _small_layer()
    full = O.moe_layer(x, w, idx, lambda e: ex[e], sh)
    ep = O.moe_layer_ep(x, w, idx, lambda e: ex[e], sh, n_experts=16, world_size=N)
    np.testing.assert_allclose(ep, full, rtol=0, atol=1e-12)


def test_partials_match_torch_per_rank():
    # rank r's share, restated with torch: its experts' weighted SwiGLU
    # outputs and the SwiGLU of its slice of the shared MLP
    x, w, idx, ex, sh = _small_layer(seed=3)
    N, E = 4, 16
    F = torch.nn.functional
    xt = torch.from_numpy(x)
    for r in range(N):
        rng_e = range(r * E // N, (r + 1) * E // N)
        f = slice(r * 32 // N, (r + 1) * 32 // N)
        ref = torch.zeros_like(xt)
        for t in range(x.shape[0]):
            for j in range(idx.shape[1]):
                e = int(idx[t, j])
                if e in rng_e:
                    w1, w3, w2 = (torch.from_numpy(a) for a in ex[e])
                    ref[t] += w[t, j] * (F.silu(xt[t] @ w1.T) * (xt[t] @ w3.T)) @ w2.T
        s1, s3, s2 = (torch.from_numpy(a) for a in sh)
        ref += (F.silu(xt @ s1[f].T) * (xt @ s3[f].T)) @ s2[:, f].T
        got = O.moe_layer_partial(x, w, idx, lambda e: ex[e], sh, expert_range=O.expert_block(E, N, r),
                                  shared_range=O.shared_block(32, N, r))
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def pin_ep_partials():
    """The share pins in one call (used by the planted-mistake tests)."""
    for N in (2, 4):
        test_partials_add_up_to_the_layer(N)
        test_expert_blocks_cover_every_expert_once(16, N)
    test_partials_match_torch_per_rank()


def test_bf16_ep_layer_within_rounding_of_the_layer():
    # with the activation roundings, the ranks round their shared slices
    # separately; the sum stays within the bf16 tolerance of the one-rank layer
    x, w, idx, ex, sh = _small_layer(seed=5)
    full = O.moe_layer(x, w, idx, lambda e: ex[e], sh, act_dtype="bf16")
    ep = O.moe_layer_ep(x, w, idx, lambda e: ex[e], sh, n_experts=16, world_size=4, act_dtype="bf16")
    scale = np.abs(full).max()
    assert (np.abs(ep - full) <= 2e-2 * np.abs(full) + 1e-2 * scale).all()
