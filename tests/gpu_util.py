"""Helpers for the GPU parity tests: device inputs from the seeded recipe, the
oracle on the same bits, the routing rule and the output tolerances.

Tolerances (stated by the layer's definition of done):
  * routing indices bit-exact for every token whose oracle margin (the
    smallest gap that decided its groups, its top-k set and their order) is
    at least 1e-6; tokens below that may differ and are then re-run through
    dispatch / experts / combine with the oracle's indices and weights;
  * routing weights within 1e-6 * route_scale (absolute);
  * fp32 layer: max |y - y_ref| <= 1e-4 * max |y_ref|;
  * bf16 layer: |y - y_ref| <= 2e-2 |y_ref| + 1e-2 max |y_ref|, per element.
"""

from __future__ import annotations

import numpy as np
import torch

from mixture_experts_layer_42_b200 import binding as M
from mixture_experts_layer_42_b200 import inputs
from oracle import moe_oracle as O

MARGIN = 1e-6


def host(t: torch.Tensor) -> np.ndarray:
    """Bits of a device tensor for the oracle (bf16 as raw uint16)."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


class Layer:
    """Device copies of one workload's inputs."""

    def __init__(self, cfg, T=None, weights=None, device="cuda"):
        self.cfg = cfg
        x, w_r, bias = inputs.routing_inputs(cfg, T)
        self.T = x.shape[0]
        self.x = x.to(device)
        self.w_r = w_r.to(device)
        self.bias = bias.to(device) if bias is not None else None
        self.bias_np = None if bias is None else bias.numpy().astype(np.float64)
        self.w = weights if weights is not None else inputs.expert_weights(cfg, device)
        self.device = device

    # ---------------------------------------------------------------- oracle
    def oracle_route(self):
        c = self.cfg
        z = O.router_logits(host(self.x), host(self.w_r))
        return O.route(z, self.bias_np, n_groups=c.n_groups, topk_groups=c.topk_groups,
                       topk=c.topk, score_func=c.score, route_scale=c.route_scale)

    def experts_np(self):
        w1, w3, w2 = self.w[:3]
        return lambda e: (host(w1[e]), host(w3[e]), host(w2[e]))

    def shared_np(self):
        ws1, ws3, ws2 = self.w[3:]
        return None if ws1 is None else (host(ws1), host(ws3), host(ws2))

    def oracle_y(self, r, tokens):
        return O.moe_layer(host(self.x), r["weights"], r["idx"], self.experts_np(), self.shared_np(),
                           act_dtype=self.cfg.dtype, tokens=tokens)

    # ---------------------------------------------------------------- GPU path
    def forward(self):
        c, T = self.cfg, self.T
        ws = M.alloc_workspace(c, T, self.device)
        y = torch.empty(T, c.dim, dtype=c.torch_dtype, device=self.device)
        wts = torch.empty(T, c.topk, dtype=torch.float32, device=self.device)
        idx = torch.empty(T, c.topk, dtype=torch.int32, device=self.device)
        w1, w3, w2, ws1, ws3, ws2 = self.w
        M.moe_forward(c, self.x, self.w_r, self.bias, w1, w3, w2, ws1, ws3, ws2, y, ws,
                      weights_out=wts, idx_out=idx)
        assert M.moe_check_error(ws) == M.MOE_OK
        return y, wts, idx

    def split(self, idx, wts, gather=False):
        """dispatch + experts + combine with the given routing (device tensors);
        with `gather`, the experts read x through src (moe_experts_grouped_gather)
        instead of an expert-contiguous copy."""
        c, T = self.cfg, self.T
        dev = self.device
        ws = M.alloc_workspace(c, T, dev)
        Tk = T * c.topk
        counts = torch.empty(c.n_routed, dtype=torch.int32, device=dev)
        offsets = torch.empty(c.n_routed + 1, dtype=torch.int32, device=dev)
        src = torch.empty(Tk, dtype=torch.int32, device=dev)
        pos = torch.empty(Tk, dtype=torch.int32, device=dev)
        x_perm = None if gather else torch.empty(Tk, c.dim, dtype=c.torch_dtype, device=dev)
        y_perm = torch.empty(Tk, c.dim, dtype=c.torch_dtype, device=dev)
        sh = c.shared_inter > 0
        s = torch.empty(T, c.dim, dtype=c.torch_dtype, device=dev) if sh else None
        y = torch.empty(T, c.dim, dtype=c.torch_dtype, device=dev)
        w1, w3, w2, ws1, ws3, ws2 = self.w
        M.moe_dispatch(c, idx, self.x, counts, offsets, src, pos, x_perm, ws)
        if gather:
            M.moe_experts_grouped_gather(c, self.x, src, offsets, w1, w3, w2, ws1, ws3, ws2, y_perm, s, ws)
        else:
            M.moe_experts_grouped(c, T, x_perm, offsets, w1, w3, w2, self.x, ws1, ws3, ws2, y_perm, s,
                                  ws)
        M.moe_combine(c, y_perm, pos, wts, s, y, ws)
        st = M.moe_check_error(ws)
        return y, dict(counts=counts, offsets=offsets, src=src, pos=pos, x_perm=x_perm,
                       y_perm=y_perm, s=s, status=st)


def check_routing(cfg, idx_gpu, w_gpu, r):
    """Apply the routing rule; returns the boolean mask of near-tie tokens whose
    GPU routing differs from the oracle's (to be re-run with the oracle's)."""
    idx_gpu = idx_gpu.cpu().numpy().astype(np.int64)
    w_gpu = w_gpu.cpu().numpy().astype(np.float64)
    differs = (idx_gpu != r["idx"]).any(axis=1)
    decided = r["margin"] >= MARGIN
    bad = np.nonzero(differs & decided)[0]
    assert len(bad) == 0, (f"{len(bad)} tokens with margin >= {MARGIN} routed differently, e.g. "
                           f"t={bad[:5].tolist()} gpu={idx_gpu[bad[:2]].tolist()} "
                           f"oracle={r['idx'][bad[:2]].tolist()} margin={r['margin'][bad[:2]].tolist()}")
    same = ~differs
    err = np.abs(w_gpu[same] - r["weights"][same]).max() if same.any() else 0.0
    assert err <= 1e-6 * cfg.route_scale, f"routing weight error {err}"
    return differs


def check_y(cfg, y_gpu_rows, y_ref):
    y = np.asarray(y_gpu_rows, dtype=np.float64)
    ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == ref.shape
    assert np.isfinite(y).all()
    scale = np.abs(ref).max()
    d = np.abs(y - ref)
    if cfg.dtype == "f32":
        assert d.max() <= 1e-4 * scale, f"max|dy| {d.max()} > 1e-4 * {scale}"
    else:
        lim = 2e-2 * np.abs(ref) + 1e-2 * scale
        worst = np.argmax(d - lim)
        assert (d <= lim).all(), (f"{int((d > lim).sum())} elements out of tolerance; worst "
                                  f"|dy|={d.flat[worst]} ref={ref.flat[worst]} max|ref|={scale}")
    return float(d.max() / scale)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def forward_parity(L: Layer, tokens=None, r=None):
    """Run the whole layer on the GPU and check it against the oracle on
    `tokens` (all when None); returns (relative max error, oracle routing)."""
    cfg = L.cfg
    y, wts, idx = L.forward()
    r = L.oracle_route() if r is None else r
    differs = check_routing(cfg, idx, wts, r)
    rows = np.arange(L.T) if tokens is None else np.asarray(tokens)
    if differs.any():
        # near-tie tokens: re-run the path with the oracle's routing
        oi = torch.from_numpy(r["idx"].astype(np.int32)).to(L.device)
        ow = torch.from_numpy(r["weights"].astype(np.float32)).to(L.device)
        y, _ = L.split(oi, ow)
    y_ref = L.oracle_y(r, rows)
    return check_y(cfg, to_np(y)[rows], y_ref), r, int(differs.sum())
