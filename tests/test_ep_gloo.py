"""The host side of the expert-parallel layer (mixture_experts_layer_42_b200.ep)
on the CPU: two and four gloo ranks each take their expert block and shared
slice with the package's partition, compute their share of y with the oracle
(the CUDA library needs a GPU; its share is checked on one GPU by
tests/test_gpu_ep.py), and sum the shares with the package's all_reduce. The
sum must equal the whole layer, and the package's partition must agree with
the oracle's (two independent statements of the pages' contiguous blocks)."""

import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

E, D, I, IS, T, K = 16, 32, 16, 32, 40, 4


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _layer():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((T, D))
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)])
    w = rng.uniform(0.1, 1.0, (T, K))
    w1 = rng.standard_normal((E, I, D)) / np.sqrt(D)
    w3 = rng.standard_normal((E, I, D)) / np.sqrt(D)
    w2 = rng.standard_normal((E, D, I)) / np.sqrt(I)
    ws1 = rng.standard_normal((IS, D)) / np.sqrt(D)
    ws3 = rng.standard_normal((IS, D)) / np.sqrt(D)
    ws2 = rng.standard_normal((D, IS)) / np.sqrt(IS)
    return x, w, idx, (w1, w3, w2, ws1, ws3, ws2)


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    from mixture_experts_layer_42_b200 import ep
    from oracle import moe_oracle as O
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        x, w, idx, weights = _layer()
        cfg = types.SimpleNamespace(n_routed=E, shared_inter=IS, dtype="f32")
        lw = ep.local_weights(cfg, tuple(torch.from_numpy(a) for a in weights), world, rank)
        b, e = ep.expert_block(E, world, rank)
        # this rank's share, from its own slices of the weights only
        share = O.moe_layer_partial(
            x, w, idx, lambda g: tuple(a[g - b].numpy() for a in lw[:3]),
            tuple(a.numpy() for a in lw[3:]), expert_range=range(b, e),
            shared_range=range(lw[3].shape[0]))
        y = ep.reduce_partial(torch.from_numpy(share).to(torch.float32))
        q.put((rank, y.numpy().astype(np.float64), (b, e), ep.shared_block(IS, world, rank, 4)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_gloo_ranks_sum_their_shares_to_the_layer(world):
    from oracle import moe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    got = sorted((q.get(timeout=180) for _ in ps), key=lambda g: g[0])
    for p in ps:
        p.join(60)
        assert p.exitcode == 0
    x, w, idx, (w1, w3, w2, ws1, ws3, ws2) = _layer()
    full = O.moe_layer(x, w, idx, lambda e: (w1[e], w3[e], w2[e]), (ws1, ws3, ws2))
    for rank, y, blk, sblk in got:
        # every rank holds the same sum after the all_reduce (fp32 shares)
        np.testing.assert_allclose(y, full, rtol=1e-5, atol=1e-5 * np.abs(full).max())
        assert range(*blk) == O.expert_block(E, world, rank)
        assert range(*sblk) == O.shared_block(IS, world, rank)


def test_partition_rejects_uneven_splits():
    sys.path.insert(0, ROOT)
    from mixture_experts_layer_42_b200 import ep
    with pytest.raises(ValueError):
        ep.expert_block(10, 4, 0)
    with pytest.raises(ValueError):
        ep.shared_block(2048, 3, 0)
    with pytest.raises(ValueError):
        ep.expert_block(16, 2, 2)
    assert ep.shared_block(0, 4, 1) == (0, 0)
    assert ep.expert_block(256, 8, 7) == (224, 256)
    assert ep.shared_block(2048, 8, 3) == (768, 1024)
