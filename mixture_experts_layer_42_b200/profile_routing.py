"""Run the layer's non-expert kernels -- router (moe_gate), dispatch
(moe_dispatch) and combine (moe_combine) -- on a workload's shapes without
allocating any expert weights, so that a profiler can capture them with a
small device footprint. The dispatched rows stand in for the expert outputs
(combine then reads rows of the same size and layout), and x stands in for
the shared expert's output.

    python -m mixture_experts_layer_42_b200.profile_routing --config v3_prefill --iters 3

Each iteration launches the six kernels once, in layer order, on one stream.
"""

from __future__ import annotations

import argparse

import torch

from . import binding as M
from . import inputs


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--config", default="v3_decode", choices=sorted(inputs.CONFIGS))
    ap.add_argument("--iters", type=int, default=3)
    a = ap.parse_args(argv)
    cfg = inputs.CONFIGS[a.config]
    T, k, D, E = cfg.T, cfg.topk, cfg.dim, cfg.n_routed
    dev = torch.device("cuda")
    x, w_r, bias = inputs.routing_inputs(cfg, T)
    x, w_r = x.to(dev), w_r.to(dev)
    bias = None if bias is None else bias.to(dev)
    wts = torch.empty(T, k, dtype=torch.float32, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    pos = torch.empty(T * k, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * k, D, dtype=x.dtype, device=dev)
    s = x if cfg.shared_inter > 0 else None
    y = torch.empty_like(x)
    ws = M.alloc_workspace(cfg, T, dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    for _ in range(a.iters):
        M.moe_gate(cfg, x, w_r, bias, wts, idx, ws, stream=stream)
        M.moe_dispatch(cfg, idx, x, counts, offsets, src, pos, x_perm, ws, stream=stream)
        M.moe_combine(cfg, x_perm, pos, wts, s, y, ws, stream=stream)
    stream.synchronize()
    st = M.moe_check_error(ws, stream=stream)
    if st != M.MOE_OK:
        raise SystemExit(f"device error word: {M.status_string(st)}")
    print(f"{cfg.name}: T={T} D={D} E={E} k={k}: {a.iters} x (gate, dispatch, combine) done; "
          f"active experts {int((counts > 0).sum())}, max count {int(counts.max())}")


if __name__ == "__main__":
    main()
