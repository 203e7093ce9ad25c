"""The FP8 expert path on the GPU, through the C ABI, against the oracle.

moe_quantize_fp8 must give the oracle's e4m3 codes and power-of-two block
scales bit for bit (128 x 128 weight blocks, 1 x 128 activation blocks).
moe_forward_fp8 is compared with the oracle's FP8 layer (the same e4m3
weights, dequantized exactly; x and h quantized per 1 x 128 block) with the
routing rule and the bf16 tolerance of the other tests. The up-projection's
h is formed in fp32 on the GPU and in fp64 by the oracle, so a value of h at
an e4m3 rounding boundary may take the neighbouring code on one side; the
tolerance covers those."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import inputs
from oracle import moe_oracle as O
from tests.gpu_util import Layer, check_routing, check_y, host, to_np

pytestmark = pytest.mark.gpu

# The two forms of the FP8 expert GEMMs: weights on the MMA's M side with up
# to 32 tokens on N (decode batches), and 128 token rows on M with 256 weight
# rows on N (large batches).
FORMS = {"tokens_on_n": M.MOE_FP8_KERNEL_TOKENS_ON_N, "tokens_on_m": M.MOE_FP8_KERNEL_TOKENS_ON_M}


@pytest.fixture(params=sorted(FORMS))
def form(request):
    M.moe_select_fp8_kernel(FORMS[request.param])
    yield request.param
    M.moe_select_fp8_kernel(M.MOE_FP8_KERNEL_AUTO)


def small(**kw):
    base = inputs.MoEConfig("fp8_small", T=300, dim=384, n_routed=16, n_groups=4, topk_groups=2,
                            topk=4, moe_inter=256, n_shared=1, score="sigmoid", bias="normal",
                            route_scale=2.5, dtype="bf16", seed=21)
    return base.with_(**kw)


def quantize(cfg, a, block_rows):
    """e4m3 codes (uint8) and scales of a [rows, cols] device tensor."""
    a2 = a.reshape(-1, a.shape[-1]).contiguous()
    R, C = a2.shape
    q = torch.empty(R, C, dtype=torch.uint8, device=a.device)
    s = torch.empty((R + block_rows - 1) // block_rows, C // 128, dtype=torch.float32, device=a.device)
    M.moe_quantize_fp8(cfg, a2, block_rows, q, s)
    return q, s


def codes(q):
    """e4m3 bytes -> float64 values."""
    return q.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


class Fp8Layer:
    """A layer's bf16 weights quantized to the FP8 layout on the GPU, with the
    dequantized weights the oracle uses."""

    def __init__(self, L):
        self.L = L
        cfg = L.cfg
        E, I, D, Is = cfg.n_routed, cfg.moe_inter, cfg.dim, cfg.shared_inter
        w1, w3, w2, ws1, ws3, ws2 = L.w
        self.q = {}
        for name, t in (("w1", w1), ("w3", w3), ("w2", w2), ("ws1", ws1), ("ws3", ws3), ("ws2", ws2)):
            if t is not None:
                self.q[name] = quantize(cfg, t, 128)
        # scales as [E, N/128, K/128] (a stacked [E*N, K] matrix has E*N/128 block rows)
        self.fw = M.fp8_weights(self.q["w1"][0], self.q["w3"][0], self.q["w2"][0],
                                self.q["w1"][1], self.q["w3"][1], self.q["w2"][1],
                                *(self.q[n][0] if n in self.q else None for n in ("ws1", "ws3", "ws2")),
                                *(self.q[n][1] if n in self.q else None for n in ("ws1", "ws3", "ws2")))
        self.shape = dict(w1=(E, I, D), w3=(E, I, D), w2=(E, D, I))

    def _deq(self, name, e=None):
        """Dequantized weights (exact: code times its block's power of two);
        for routed experts one expert at a time, as the oracle asks for them."""
        q, s = self.q[name]
        if e is not None:
            _, n, k = self.shape[name]
            q = q[e * n:(e + 1) * n]
            s = s[e * n // 128:(e + 1) * n // 128]
        return O.dequantize_blocks(codes(q), s.cpu().numpy().astype(np.float64), 128, 128)

    def experts(self):
        return lambda e: tuple(self._deq(n, e) for n in ("w1", "w3", "w2"))

    def shared(self):
        if "ws1" not in self.q:
            return None
        return tuple(self._deq(n) for n in ("ws1", "ws3", "ws2"))

    def forward(self):
        L, cfg = self.L, self.L.cfg
        ws = M.alloc_workspace_fp8(cfg, L.T)
        y = torch.empty(L.T, cfg.dim, dtype=torch.bfloat16, device="cuda")
        wts = torch.empty(L.T, cfg.topk, dtype=torch.float32, device="cuda")
        idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
        M.moe_forward_fp8(cfg, L.x, L.w_r, L.bias, self.fw, y, ws, weights_out=wts, idx_out=idx)
        assert M.moe_check_error(ws) == M.MOE_OK
        return y, wts, idx


@pytest.mark.parametrize("block_rows,shape", [(128, (512, 384)), (128, (300, 256)), (1, (77, 7168)),
                                              (1, (5, 128))])
def test_quantizer_matches_the_oracle_bitwise(block_rows, shape):
    cfg = small()
    g = torch.Generator().manual_seed(shape[0])
    a = (torch.randn(*shape, generator=g) * torch.exp(torch.randn(shape[0], 1, generator=g))).to(torch.bfloat16)
    q, s = quantize(cfg, a.cuda(), block_rows)
    oq, os_ = O.quantize_blocks(host(a), block_rows, 128)
    np.testing.assert_array_equal(codes(q), oq)
    np.testing.assert_array_equal(s.cpu().numpy().astype(np.float64), os_)


def test_quantizer_on_zero_and_extreme_blocks():
    cfg = small()
    a = torch.zeros(256, 256, dtype=torch.bfloat16)
    a[128:, 128:] = 3.0e38                      # a block at the top of bf16's range
    a[0, 128] = 2.0 ** -120                     # a block of one tiny value
    q, s = quantize(cfg, a.cuda(), 128)
    oq, os_ = O.quantize_blocks(host(a), 128, 128)
    np.testing.assert_array_equal(codes(q), oq)
    np.testing.assert_array_equal(s.cpu().numpy().astype(np.float64), os_)


def _parity(cfg):
    L = Layer(cfg)
    F = Fp8Layer(L)
    y, wts, idx = F.forward()
    r = L.oracle_route()
    differs = check_routing(cfg, idx, wts, r)
    rows = np.nonzero(~differs)[0]
    yref = O.moe_layer(host(L.x), r["weights"], r["idx"], F.experts(), F.shared(), act_dtype="bf16",
                       tokens=rows, fp8=True)
    return check_y(cfg, to_np(y)[rows], yref), L, F, y


@pytest.mark.parametrize("kw", [{}, dict(T=1), dict(T=77), dict(T=129, moe_inter=128, dim=256),
                                dict(n_shared=0), dict(n_routed=64, n_groups=8, topk_groups=3, topk=6),
                                dict(T=1000, n_routed=8, n_groups=2, topk_groups=1, topk=2),
                                dict(score="softmax", bias="none", n_groups=1, topk_groups=1, n_shared=2)])
def test_fp8_forward_matches_oracle(kw, form):
    err, *_ = _parity(small(**kw))
    assert err < 2e-2


@pytest.mark.parametrize("kw", [dict(T=2048, n_routed=8, n_groups=2, topk_groups=1, topk=2, dim=512,
                                     moe_inter=384),
                                dict(T=700, n_routed=4, n_groups=1, topk_groups=1, topk=1, n_shared=0),
                                dict(T=513, dim=256, moe_inter=128, n_routed=2, n_groups=1,
                                     topk_groups=1, topk=2),
                                dict(T=600, dim=128, moe_inter=128, n_routed=4, n_groups=1,
                                     topk_groups=1, topk=2),
                                dict(T=300, dim=8192, moe_inter=256, n_routed=4, n_groups=1,
                                     topk_groups=1, topk=2)])
def test_fp8_forward_many_rows_per_expert(kw, form):
    # experts with several 128-row tiles and ragged last tiles; a layer with
    # dim an odd multiple of 128 (its last down-projection tile one weight
    # block wide); every expert taking every token; the smallest and the
    # largest reduction depth the FP8 layout allows (one 128-deep k-block,
    # and 64 of them)
    err, *_ = _parity(small(**kw))
    assert err < 2e-2


def test_fp8_forward_v3_decode_all_tokens():
    # the DeepSeek-V3 decode batch with its weights in the FP8 layout
    err, L, F, y = _parity(inputs.CONFIGS["v3_decode"])
    assert err < 2e-2
    # and within the quantization noise of the bf16 layer
    y16, _, _ = L.forward()
    a, b = to_np(y), to_np(y16)
    assert np.abs(a - b).max() <= 0.1 * np.abs(b).max()


def test_fp8_shapes_are_checked():
    cfg = small(moe_inter=192)                  # not a multiple of 128
    with pytest.raises(M.MoEError) as e:
        M.moe_workspace_size_fp8(cfg, 64)
    assert e.value.status == M.MOE_ERR_UNSUPPORTED
    with pytest.raises(M.MoEError) as e:
        M.moe_workspace_size_fp8(inputs.CONFIGS["tiny_fp32"], 64)
    assert e.value.status == M.MOE_ERR_UNSUPPORTED


def test_fp8_forward_with_zero_and_tiny_rows(form):
    # a token row of zeros (its blocks' scale 2^0, UE8M0 byte 127) and rows so
    # small that their blocks take the smallest scale, 2^-127 (UE8M0 byte 0),
    # through the block-scaled forward, against the oracle's FP8 layer
    cfg = small(T=64)
    L = Layer(cfg)
    x = L.x.float()
    x[0] = 0.0
    x[1:4] = x[1:4] * 2.0 ** -125
    L.x = x.to(torch.bfloat16).contiguous()
    xq, xs = quantize(cfg, L.x, 1)
    s = xs.cpu().numpy()
    assert (s[0] == 1.0).all() and (s[1:4] == 2.0 ** -127).mean() > 0.5
    F = Fp8Layer(L)
    y, wts, idx = F.forward()
    r = L.oracle_route()
    differs = check_routing(cfg, idx, wts, r)
    rows = np.nonzero(~differs)[0]
    assert {0, 1, 2, 3} <= set(rows.tolist())
    yref = O.moe_layer(host(L.x), r["weights"], r["idx"], F.experts(), F.shared(), act_dtype="bf16",
                       tokens=rows, fp8=True)
    assert check_y(cfg, to_np(y)[rows], yref) < 2e-2


@pytest.mark.slow
def test_fp8_forward_v3_prefill_sampled_tokens():
    # the DeepSeek-V3 prefill batch (T = 8192) with its weights in the FP8
    # layout, in the form the layer picks for it (tokens on M): routing on
    # every token, outputs on a seeded sample that includes tokens of the most
    # and least loaded experts and the first and last token
    cfg = inputs.CONFIGS["v3_prefill"]
    L = Layer(cfg)
    F = Fp8Layer(L)
    y, wts, idx = F.forward()
    r = L.oracle_route()
    differs = check_routing(cfg, idx, wts, r)
    rng = np.random.default_rng(11)
    counts = np.bincount(r["idx"].ravel(), minlength=cfg.n_routed)
    hot, cold = int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))
    picks = [np.nonzero((r["idx"] == hot).any(1))[0][:3], np.nonzero((r["idx"] == cold).any(1))[0][:3],
             [0, L.T - 1], rng.choice(L.T, 40, replace=False)]
    tokens = np.unique(np.concatenate(picks))
    tokens = tokens[~differs[tokens]]
    yref = O.moe_layer(host(L.x), r["weights"], r["idx"], F.experts(), F.shared(), act_dtype="bf16",
                       tokens=tokens, fp8=True)
    assert check_y(cfg, to_np(y)[tokens], yref) < 2e-2


def test_fp8_forward_replays_from_a_cuda_graph(form):
    # moe_forward_fp8 does no host synchronisation and allocates nothing: it
    # can be captured once and replayed with new token rows written into the
    # same buffer, giving what an eager call gives on those rows
    cfg = small(T=700, n_routed=8, n_groups=2, topk_groups=1, topk=2)
    L = Layer(cfg)
    F = Fp8Layer(L)
    ws = M.alloc_workspace_fp8(cfg, L.T)
    y = torch.empty(L.T, cfg.dim, dtype=torch.bfloat16, device="cuda")
    x = L.x.clone()
    s = torch.cuda.Stream()

    def run():
        M.moe_forward_fp8(cfg, x, L.w_r, L.bias, F.fw, y, ws, stream=s)

    with torch.cuda.stream(s):
        run()                                   # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    gen = torch.Generator().manual_seed(12)
    for _ in range(3):
        x.copy_(torch.randn(L.T, cfg.dim, generator=gen).to(torch.bfloat16).cuda())
        g.replay()
        torch.cuda.synchronize()
        got = y.clone()
        with torch.cuda.stream(s):
            run()                               # the same rows, eagerly
        torch.cuda.synchronize()
        assert torch.equal(got, y)
        assert M.moe_check_error(ws) == M.MOE_OK
