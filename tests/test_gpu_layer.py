"""GPU parity of the layer's steps and of the whole layer against the oracle,
on small and medium shapes and the edge cases (runs through the C ABI)."""

import numpy as np
import pytest
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import inputs
from oracle import moe_oracle as O
from tests.gpu_util import Layer, check_routing, check_y, forward_parity, host, to_np

pytestmark = pytest.mark.gpu

TINY = inputs.CONFIGS["tiny_fp32"]


def bf16_small(**kw):
    """A bf16 layer small enough for the full oracle, spanning several
    128-row tiles, ragged feature tiles and a ragged token tail."""
    base = inputs.MoEConfig("bf16_small", T=300, dim=384, n_routed=16, n_groups=4, topk_groups=2,
                            topk=4, moe_inter=192, n_shared=1, score="sigmoid", bias="normal",
                            route_scale=2.5, dtype="bf16", seed=3)
    return base.with_(**kw)


# ---------------------------------------------------------------- whole layer

def test_tiny_fp32_forward_all_tokens():
    err, r, nt = forward_parity(Layer(TINY))
    assert err < 1e-4


@pytest.mark.parametrize("kw", [
    {},
    dict(T=1),
    dict(T=77),
    dict(T=129, dim=256, moe_inter=128),
    dict(score="softmax", bias="none", n_groups=1, topk_groups=1, topk=6, n_routed=64, n_shared=2),
    dict(n_routed=64, n_groups=8, topk_groups=3, topk=6, moe_inter=136),
    dict(n_shared=0),
    dict(T=513, dim=1024, moe_inter=512, n_routed=32, n_groups=4, topk_groups=2, topk=8),
    # the most experts and picks the library accepts: 1024 experts, top-32
    dict(T=200, dim=256, moe_inter=128, n_routed=1024, n_groups=32, topk_groups=8, topk=32),
])
def test_bf16_forward_all_tokens(kw):
    err, r, nt = forward_parity(Layer(bf16_small(**kw)))
    assert err < 2e-2


@pytest.mark.parametrize("kw", [dict(T=1), dict(T=100, score="softmax", bias="none", n_groups=1,
                                                  topk_groups=1), dict(n_shared=2, T=200)])
def test_fp32_forward_variants(kw):
    err, r, nt = forward_parity(Layer(TINY.with_(**kw)))
    assert err < 1e-4


def test_softmax_nogroup_all_tokens():
    # the softmax workload at full size (T = 4096, D = 2048, 64 experts,
    # top-6, two shared experts), every token against the oracle
    err, r, nt = forward_parity(Layer(inputs.CONFIGS["softmax_nogroup"]))
    assert err < 2e-2


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("name", ["tiny_fp32", "v3_decode", "softmax_nogroup", "v3_prefill", "v3_zipf"])
def test_gate_all_tokens(name):
    cfg = inputs.CONFIGS[name]
    L = Layer(cfg, weights=(None,) * 6)
    wts = torch.empty(L.T, cfg.topk, dtype=torch.float32, device="cuda")
    idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg, L.T)
    M.moe_gate(cfg, L.x, L.w_r, L.bias, wts, idx, ws)
    torch.cuda.synchronize()
    r = L.oracle_route()
    differs = check_routing(cfg, idx, wts, r)
    assert differs.sum() <= max(2, L.T // 1000)


@pytest.mark.parametrize("kw", [
    # the largest routing shapes the library accepts, and unusual group widths
    dict(n_routed=1024, n_groups=32, topk_groups=8, topk=32),            # 32 experts per group
    dict(n_routed=1024, n_groups=64, topk_groups=16, topk=8),            # 16 per group
    dict(n_routed=1024, n_groups=1, topk_groups=1, topk=32, score="softmax", bias="none"),
    dict(n_routed=8, n_groups=4, topk_groups=2, topk=4),                 # 2 per group (top-2 = both)
    dict(n_routed=96, n_groups=3, topk_groups=2, topk=6),                # E not a power of two
    dict(n_routed=48, n_groups=3, topk_groups=1, topk=16),               # k = the whole kept group
    dict(n_routed=512, n_groups=8, topk_groups=4, topk=1),               # k = 1
    dict(n_routed=64, n_groups=2, topk_groups=2, topk=8),                # every group kept
])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_gate_routing_limits(kw, dtype):
    cfg = bf16_small(T=333, dim=512, dtype=dtype, **kw)
    L = Layer(cfg, weights=(None,) * 6)
    wts = torch.empty(L.T, cfg.topk, dtype=torch.float32, device="cuda")
    idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg, L.T)
    M.moe_gate(cfg, L.x, L.w_r, L.bias, wts, idx, ws)
    torch.cuda.synchronize()
    r = L.oracle_route()
    differs = check_routing(cfg, idx, wts, r)
    assert differs.sum() <= 2


def test_gate_zero_router_closed_form():
    # W_r = 0: all scores 0.5, selection by the bias alone, weights route_scale / k
    cfg = bf16_small(T=50)
    L = Layer(cfg, weights=(None,) * 6)
    L.w_r.zero_()
    bias = torch.zeros(cfg.n_routed)
    bias[[5, 6]] = torch.tensor([0.30, 0.20])
    bias[[12, 15]] = torch.tensor([0.25, 0.10])
    bias[0] = 0.28
    L.bias = bias.cuda()
    wts = torch.empty(L.T, cfg.topk, dtype=torch.float32, device="cuda")
    idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg, L.T)
    M.moe_gate(cfg, L.x, L.w_r, L.bias, wts, idx, ws)
    assert (idx.cpu() == torch.tensor([5, 12, 6, 15], dtype=torch.int32)).all()
    assert (wts.cpu() == cfg.route_scale / cfg.topk).all()


def test_gate_softmax_ties_lowest_index():
    cfg = bf16_small(T=20, score="softmax", bias="none", n_groups=1, topk_groups=1, n_routed=64, topk=6)
    L = Layer(cfg, weights=(None,) * 6)
    L.w_r.zero_()
    wts = torch.empty(L.T, cfg.topk, dtype=torch.float32, device="cuda")
    idx = torch.empty(L.T, cfg.topk, dtype=torch.int32, device="cuda")
    ws = M.alloc_workspace(cfg, L.T)
    M.moe_gate(cfg, L.x, L.w_r, None, wts, idx, ws)
    assert (idx.cpu() == torch.arange(6, dtype=torch.int32)).all()
    np.testing.assert_allclose(wts.cpu().numpy(), cfg.route_scale / 64, rtol=1e-6)


# ---------------------------------------------------------------- dispatch

def _dispatch_check(L, idx_np, out):
    d = O.dispatch(idx_np, L.cfg.n_routed)
    assert (out["counts"].cpu().numpy() == d["counts"]).all()
    assert (out["offsets"].cpu().numpy() == d["offsets"]).all()
    assert (out["src"].cpu().numpy() == d["src"]).all()
    assert (out["pos"].cpu().numpy().reshape(idx_np.shape) == d["pos"]).all()
    if out.get("x_perm") is not None:
        xp = out["x_perm"].cpu()
        assert torch.equal(xp, L.x.cpu()[torch.from_numpy(d["src"])])


@pytest.mark.parametrize("copy_rows", [True, False], ids=["x_perm", "indices_only"])
@pytest.mark.parametrize("name,T", [("tiny_fp32", None), ("v3_decode", None), ("v3_zipf", 2048)])
def test_dispatch_matches_oracle(name, T, copy_rows):
    cfg = inputs.CONFIGS[name]
    L = Layer(cfg, T=T, weights=(None,) * 6)
    r = L.oracle_route()
    idx = torch.from_numpy(r["idx"].astype(np.int32)).cuda()
    w = torch.from_numpy(r["weights"].astype(np.float32)).cuda()
    # experts are not needed for dispatch: run dispatch alone
    c = cfg
    Tk = L.T * c.topk
    ws = M.alloc_workspace(c, L.T)
    out = dict(counts=torch.empty(c.n_routed, dtype=torch.int32, device="cuda"),
               offsets=torch.empty(c.n_routed + 1, dtype=torch.int32, device="cuda"),
               src=torch.empty(Tk, dtype=torch.int32, device="cuda"),
               pos=torch.empty(Tk, dtype=torch.int32, device="cuda"),
               x_perm=torch.empty(Tk, c.dim, dtype=c.torch_dtype, device="cuda") if copy_rows else None)
    M.moe_dispatch(c, idx, L.x if copy_rows else None, out["counts"], out["offsets"], out["src"],
                   out["pos"], out["x_perm"], ws)
    assert M.moe_check_error(ws) == M.MOE_OK
    _dispatch_check(L, r["idx"], out)


@pytest.mark.parametrize("T,E,k,bad", [(1, 8, 2, False), (128, 256, 8, False), (512, 512, 8, False),
                                       (4096, 16, 1, False), (300, 64, 6, True)])
def test_one_kernel_dispatch_equals_the_chunked_dispatch(T, E, k, bad):
    # small batches without the row copy take one kernel (one CTA): the same
    # counts, offsets, pos and src, bit for bit, as the chunked three-kernel
    # path that the copy takes (the largest case is exactly 4096 pairs)
    cfg = bf16_small(T=T, n_routed=E, n_groups=1, topk_groups=1, topk=k, dim=128, n_shared=0)
    g = torch.Generator().manual_seed(T + E)
    idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
    if bad:
        idx[7, 2] = E + 3            # out of range: flagged, its pair dropped
        idx[11, 0] = -1
    idx = idx.cuda()
    x = torch.randn(T, cfg.dim, generator=g).to(torch.bfloat16).cuda()
    outs = []
    for copy in (True, False):
        ws = M.alloc_workspace(cfg, T)
        o = [torch.full((n,), -7, dtype=torch.int32, device="cuda") for n in (E, E + 1, T * k, T * k)]
        xp = torch.empty(T * k, cfg.dim, dtype=torch.bfloat16, device="cuda") if copy else None
        M.moe_dispatch(cfg, idx, x if copy else None, *o, xp, ws)
        status = M.moe_check_error(ws)
        assert status == (M.MOE_ERR_DEVICE_CHECK if bad else M.MOE_OK)
        outs.append(o)
    n_valid = int(outs[0][1][E].item())
    for a, b, name in zip(outs[0], outs[1], ("counts", "offsets", "src", "pos")):
        if name == "src":            # rows past the valid pairs are not written
            a, b = a[:n_valid], b[:n_valid]
        assert torch.equal(a, b), name


def test_dispatch_all_tokens_same_experts():
    # extreme skew: every token picks experts {3, 7, 9, 12}
    cfg = bf16_small(T=1000)
    L = Layer(cfg, weights=(None,) * 6)
    idx_np = np.tile(np.array([[9, 3, 12, 7]]), (L.T, 1))
    out = {}
    Tk = L.T * 4
    ws = M.alloc_workspace(cfg, L.T)
    for k_, n in (("counts", 16), ("offsets", 17), ("src", Tk), ("pos", Tk)):
        out[k_] = torch.empty(n, dtype=torch.int32, device="cuda")
    out["x_perm"] = torch.empty(Tk, cfg.dim, dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(cfg, torch.from_numpy(idx_np.astype(np.int32)).cuda(), L.x, out["counts"],
                   out["offsets"], out["src"], out["pos"], out["x_perm"], ws)
    _dispatch_check(L, idx_np, out)


def test_dispatch_bad_index_flagged_and_dropped():
    cfg = bf16_small(T=64)
    L = Layer(cfg, weights=(None,) * 6)
    r = L.oracle_route()
    idx_np = r["idx"].copy()
    idx_np[5, 1] = cfg.n_routed + 3
    idx_np[17, 0] = -1
    Tk = L.T * cfg.topk
    ws = M.alloc_workspace(cfg, L.T)
    counts = torch.empty(16, dtype=torch.int32, device="cuda")
    offsets = torch.empty(17, dtype=torch.int32, device="cuda")
    src = torch.full((Tk,), -7, dtype=torch.int32, device="cuda")
    pos = torch.empty(Tk, dtype=torch.int32, device="cuda")
    x_perm = torch.zeros(Tk, cfg.dim, dtype=torch.bfloat16, device="cuda")
    M.moe_dispatch(cfg, torch.from_numpy(idx_np.astype(np.int32)).cuda(), L.x, counts, offsets, src,
                   pos, x_perm, ws)
    assert M.moe_check_error(ws) == M.MOE_ERR_DEVICE_CHECK
    assert M.moe_check_error(ws) == M.MOE_OK          # the error word was cleared
    assert offsets[-1].item() == Tk - 2
    p = pos.cpu().numpy().reshape(L.T, cfg.topk)
    assert p[5, 1] == -1 and p[17, 0] == -1
    assert (src.cpu().numpy()[Tk - 2:] == -7).all()   # nothing written past the valid rows
    good = idx_np.copy()
    assert counts.sum().item() == Tk - 2


# ---------------------------------------------------------------- experts

def _experts_case(cfg):
    L = Layer(cfg)
    r = L.oracle_route()
    idx = torch.from_numpy(r["idx"].astype(np.int32)).cuda()
    w = torch.from_numpy(r["weights"].astype(np.float32)).cuda()
    return L, r, idx, w


class _kernel:
    """Select the GEMM kernels for the duration of a block."""

    def __init__(self, which):
        self.which = which

    def __enter__(self):
        M.moe_select_expert_kernel(self.which)

    def __exit__(self, *exc):
        M.moe_select_expert_kernel(M.MOE_EXPERT_KERNEL_AUTO)


TC_KERNELS = [M.MOE_EXPERT_KERNEL_TCGEN05, M.MOE_EXPERT_KERNEL_TCGEN05_PAIR]


@pytest.mark.parametrize("which", TC_KERNELS, ids=["one_cta", "cta_pair"])
@pytest.mark.parametrize("kw", [{}, dict(T=640, dim=512, moe_inter=256), dict(moe_inter=200),
                                dict(T=2000, n_routed=8, n_groups=2, topk_groups=1, topk=2),
                                dict(T=200, dim=256, moe_inter=128, n_routed=1024, n_groups=32,
                                     topk_groups=8, topk=32)])
def test_tensor_core_experts_match_oracle(kw, which):
    cfg = bf16_small(**kw)
    L, r, idx, w = _experts_case(cfg)
    with _kernel(which):
        y, out = L.split(idx, w)
    assert out["status"] == M.MOE_OK
    d = O.dispatch(r["idx"], cfg.n_routed)
    xp = host(out["x_perm"])
    yp = to_np(out["y_perm"])
    w1, w3, w2 = L.w[:3]
    for e in range(cfg.n_routed):
        a, b = d["offsets"][e], d["offsets"][e + 1]
        if a == b:
            continue
        ref = O.swiglu(xp[a:b], host(w1[e]), host(w3[e]), host(w2[e]), round_h="bf16", round_out="bf16")
        check_y(cfg, yp[a:b], ref)
    ws1, ws3, ws2 = L.w[3:]
    sref = O.swiglu(host(L.x), host(ws1), host(ws3), host(ws2), round_h="bf16", round_out="bf16")
    check_y(cfg, to_np(out["s"]), sref)


@pytest.mark.parametrize("kw", [dict(T=640, dim=512, moe_inter=256),
                                dict(T=256, dim=7168, moe_inter=2048, n_routed=16, topk=8,
                                     n_groups=4, topk_groups=4)])
def test_tensor_core_vs_simt(kw):
    # two independent GPU kernels for the same grouped GEMM; both accumulate in
    # fp32, so they agree far tighter than the layer tolerance
    cfg = bf16_small(**kw)
    L, r, idx, w = _experts_case(cfg)
    with _kernel(M.MOE_EXPERT_KERNEL_SIMT):
        y_si, out_si = L.split(idx, w)
    b = to_np(out_si["y_perm"])
    scale = np.abs(b).max()
    for which in TC_KERNELS:
        with _kernel(which):
            y_tc, out_tc = L.split(idx, w)
        a = to_np(out_tc["y_perm"])
        assert np.abs(a - b).max() <= 2e-2 * scale
        rel = np.abs(a - b) / (np.abs(b) + 1e-2 * scale)
        assert np.median(rel) < 1e-2


@pytest.mark.parametrize("which", [M.MOE_EXPERT_KERNEL_TCGEN05, M.MOE_EXPERT_KERNEL_SIMT],
                         ids=["tensor_core", "cuda_core"])
@pytest.mark.parametrize("kw", [{}, dict(T=77), dict(T=640, dim=512, moe_inter=256),
                                dict(T=2000, n_routed=8, n_groups=2, topk_groups=1, topk=2),
                                dict(T=200, dim=256, moe_inter=128, n_routed=1024, n_groups=32,
                                     topk_groups=8, topk=32),
                                dict(n_shared=0)])
def test_gathered_rows_match_the_permuted_copy_bitwise(kw, which):
    # the experts reading x through src (tile::gather4 on the tensor cores)
    # see the same A rows as with the expert-contiguous copy, padding rows
    # included (zeros both ways), so every output is bit for bit the same
    cfg = bf16_small(**kw)
    L, r, idx, w = _experts_case(cfg)
    with _kernel(which):
        y_c, out_c = L.split(idx, w)
        y_g, out_g = L.split(idx, w, gather=True)
    assert out_c["status"] == M.MOE_OK and out_g["status"] == M.MOE_OK
    assert torch.equal(y_c, y_g)
    assert torch.equal(out_c["y_perm"], out_g["y_perm"])
    if cfg.n_shared:
        assert torch.equal(out_c["s"], out_g["s"])
    err = check_y(cfg, to_np(y_g), L.oracle_y(r, np.arange(L.T)))
    assert err < 2e-2


def test_gathered_experts_need_the_one_cta_kernel():
    cfg = bf16_small(T=64)
    L, r, idx, w = _experts_case(cfg)
    with _kernel(M.MOE_EXPERT_KERNEL_TCGEN05_PAIR):
        with pytest.raises(M.MoEError) as e:
            L.split(idx, w, gather=True)
    assert e.value.status == M.MOE_ERR_UNSUPPORTED


def test_forward_on_the_cta_pair_kernel():
    # moe_forward on the CTA-pair option dispatches an expert-contiguous copy
    # of x into y_perm's space, which the down-projection then overwrites
    cfg = bf16_small(T=700, dim=512, moe_inter=256)
    with _kernel(M.MOE_EXPERT_KERNEL_TCGEN05_PAIR):
        err, r, nt = forward_parity(Layer(cfg))
    assert err < 2e-2


def test_pair_and_single_cta_kernels_agree_bitwise():
    # the two tensor-core kernels add the same products in the same k order
    # into fp32 accumulators, so their bf16 outputs are identical
    cfg = bf16_small(T=1500, dim=512, moe_inter=256, n_routed=8, n_groups=2, topk_groups=1, topk=2)
    L, r, idx, w = _experts_case(cfg)
    outs = []
    for which in TC_KERNELS:
        with _kernel(which):
            y, out = L.split(idx, w)
        outs.append((y.cpu(), out["y_perm"].cpu(), out["s"].cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_identity_experts_closed_form_gpu():
    # I = D, w1 = w3 = Id, w2 = c_e Id (c_e powers of two) and no shared MLP:
    # y_d = sum_j w_j c_{idx_j} * round(x_d^2 sigmoid(x_d))
    cfg = bf16_small(T=200, dim=128, moe_inter=128, n_shared=0)
    L = Layer(cfg)
    E, D = cfg.n_routed, cfg.dim
    eye = torch.eye(D, dtype=torch.bfloat16, device="cuda")
    c = 2.0 ** (np.arange(E) % 4)
    L.w = (eye.expand(E, D, D).contiguous(), eye.expand(E, D, D).contiguous(),
           torch.stack([float(c[e]) * eye for e in range(E)]).contiguous(), None, None, None)
    y, wts, idx = L.forward()
    x = host(L.x)
    xf = O.to_f64(x)
    h = O.round_bf16(xf * xf / (1 + np.exp(-xf)))
    ii, ww = idx.cpu().numpy(), wts.cpu().numpy().astype(np.float64)
    ref = (ww * c[ii]).sum(-1, keepdims=True) * h
    check_y(cfg, to_np(y), O.round_bf16(ref))


def test_zero_w1_gives_shared_only_gpu():
    cfg = bf16_small(T=100)
    L = Layer(cfg)
    L.w = (torch.zeros_like(L.w[0]),) + tuple(L.w[1:])
    y, wts, idx = L.forward()
    ws1, ws3, ws2 = L.w[3:]
    sref = O.swiglu(host(L.x), host(ws1), host(ws3), host(ws2), round_h="bf16", round_out="bf16")
    check_y(cfg, to_np(y), sref)


@pytest.mark.parametrize("layout", ["w3_below_w1", "w1_is_w3", "one_buffer"])
def test_w1_w3_memory_layouts(layout):
    # the up-projection loads the w1 and w3 tiles with one TMA box over both
    # tensors when their distance allows it, in either address order, and
    # with two boxes otherwise: all three must give the oracle's layer
    cfg = bf16_small(T=400)
    L = Layer(cfg)
    w1, w3, w2, ws1, ws3, ws2 = L.w
    if layout == "w3_below_w1":
        buf = torch.empty((2,) + tuple(w1.shape), dtype=w1.dtype, device="cuda")
        buf[0].copy_(w3)
        buf[1].copy_(w1)
        sbuf = torch.empty((2,) + tuple(ws1.shape), dtype=ws1.dtype, device="cuda")
        sbuf[0].copy_(ws3)
        sbuf[1].copy_(ws1)
        L.w = (buf[1], buf[0], w2, sbuf[1], sbuf[0], ws2)
    elif layout == "w1_is_w3":
        L.w = (w1, w1, w2, ws1, ws1, ws2)
    else:  # w1 and w3 adjacent in one allocation, w1 first
        buf = torch.stack([w1, w3])
        L.w = (buf[0], buf[1], w2, ws1, ws3, ws2)
    err, r, nt = forward_parity(L)
    assert err < 2e-2


@pytest.mark.parametrize("name", ["tiny_fp32", "softmax_nogroup"])
def test_bench_routing_only_mode_runs(name, capsys):
    # the benchmark's mode for profiling the non-expert kernels (no expert weights)
    import bench
    bench.main(["--routing-only", "--config", name, "--iters", "2"])
    assert "done" in capsys.readouterr().out


def test_stage_timing_records_one_call_in_every():
    L = Layer(bf16_small())
    M.moe_stage_timing_begin_every(3, 2)       # calls 0, 2, 4 of the next seven
    for _ in range(7):
        L.forward()
    n, ms = M.moe_stage_timing_end()
    assert n == 3
    assert all(v >= 0 for v in ms.values()) and ms["experts_up"] > 0
    M.moe_stage_timing_begin(4)                # every call, up to four
    for _ in range(5):
        L.forward()
    n, ms = M.moe_stage_timing_end()
    assert n == 4 and ms["router_logits"] > 0


@pytest.mark.parametrize("kw", [dict(T=64), dict(T=1500)], ids=["one_kernel_dispatch", "chunked_dispatch"])
def test_back_to_back_forwards_on_one_stream(kw):
    # the forward's kernels are chained as programmatic dependent launches:
    # eight forwards issued back to back on one stream, x rewritten on the
    # stream between them and no host synchronisation, must each give the
    # output of that x run alone
    cfg = bf16_small(**kw)
    L = Layer(cfg)
    w1, w3, w2, ws1, ws3, ws2 = L.w
    gen = torch.Generator().manual_seed(5)
    xs = [torch.randn(L.T, cfg.dim, generator=gen).to(cfg.torch_dtype).cuda() for _ in range(8)]
    ws = M.alloc_workspace(cfg, L.T)
    x = torch.empty_like(L.x)
    refs = []
    for xi in xs:
        x.copy_(xi)
        y = torch.empty(L.T, cfg.dim, dtype=cfg.torch_dtype, device="cuda")
        M.moe_forward(cfg, x, L.w_r, L.bias, w1, w3, w2, ws1, ws3, ws2, y, ws)
        torch.cuda.synchronize()
        refs.append(y)
    s = torch.cuda.Stream()
    ys = [torch.empty_like(r) for r in refs]
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for xi, y in zip(xs, ys):
            x.copy_(xi)
            M.moe_forward(cfg, x, L.w_r, L.bias, w1, w3, w2, ws1, ws3, ws2, y, ws, stream=s)
    torch.cuda.synchronize()
    assert M.moe_check_error(ws) == M.MOE_OK
    for y, r in zip(ys, refs):
        assert torch.equal(y, r)


def test_forward_replays_from_a_cuda_graph():
    # moe_forward does no host synchronisation and allocates nothing, so it can
    # be captured once and replayed with new inputs written into the same buffers
    cfg = bf16_small(T=300)
    L = Layer(cfg)
    ws = M.alloc_workspace(cfg, L.T)
    y = torch.empty(L.T, cfg.dim, dtype=cfg.torch_dtype, device="cuda")
    x = L.x.clone()
    w1, w3, w2, ws1, ws3, ws2 = L.w
    s = torch.cuda.Stream()

    def run():
        M.moe_forward(cfg, x, L.w_r, L.bias, w1, w3, w2, ws1, ws3, ws2, y, ws, stream=s)

    with torch.cuda.stream(s):
        run()                                   # warm-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run()
    gen = torch.Generator().manual_seed(11)
    for _ in range(3):
        xi = torch.randn(L.T, cfg.dim, generator=gen).to(cfg.torch_dtype)
        x.copy_(xi.cuda())
        g.replay()
        torch.cuda.synchronize()
        got = y.clone()
        with torch.cuda.stream(s):
            run()                               # the same inputs, eagerly
        torch.cuda.synchronize()
        assert torch.equal(got, y)
        assert M.moe_check_error(ws) == M.MOE_OK
