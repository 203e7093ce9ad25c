"""Expert parallelism of the MoE layer over the GPUs of one node.

The partition is the pages' own (the MoE class on the hackaday page and
DeepseekV3MoE.__init__ on the thataiguy page): rank r of world_size holds the
contiguous block of n_routed / world_size experts starting at
r * n_routed / world_size. Every rank routes every token (the gate is
replicated), runs only its own experts, and one all_reduce sums the ranks'
outputs. The V3.2 listing on page "Weighted expert sum" adds the shared MLP
into y before that all_reduce, so each rank also holds a contiguous slice of
the shared MLP's inner width (rows of ws1 and ws3, columns of ws2); the
slices' outputs add up to the whole MLP because each inner feature
contributes independently.

Per step and rank: moe_forward_ep (router, dispatch, this rank's grouped
experts and shared slice, and a combine into an fp32 share of y), one
all_reduce of that share (fp32 sum, the accumulator dtype of the layer), and
moe_cast_output (the single cast back to the activation dtype). The share is
T x D fp32 per rank; over NVLink 5 the all_reduce of the V3 prefill batch
(235 MB) is the exchange step.
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch


def expert_block(n_routed: int, world_size: int, rank: int) -> Tuple[int, int]:
    """[begin, end) of the experts held by `rank`."""
    if world_size < 1 or not 0 <= rank < world_size:
        raise ValueError("rank must lie in [0, world_size)")
    if n_routed % world_size:
        raise ValueError(f"{n_routed} experts do not divide over {world_size} ranks")
    per = n_routed // world_size
    return rank * per, (rank + 1) * per


def shared_block(shared_inter: int, world_size: int, rank: int, align: int = 8) -> Tuple[int, int]:
    """[begin, end) of the shared MLP's inner features held by `rank`; each
    slice is a multiple of `align` features (16-byte rows of bf16)."""
    if shared_inter == 0:
        return 0, 0
    if world_size < 1 or not 0 <= rank < world_size:
        raise ValueError("rank must lie in [0, world_size)")
    if shared_inter % (world_size * align):
        raise ValueError(f"a shared width of {shared_inter} does not split into {world_size} "
                         f"slices of a multiple of {align}")
    per = shared_inter // world_size
    return rank * per, (rank + 1) * per


def local_weights(cfg, w, world_size: int, rank: int):
    """This rank's expert weights and shared slice, as contiguous tensors on
    the device of `w`: (w1, w3, w2) of its expert block and (ws1, ws3, ws2)
    of its shared slice (None when the layer has no shared MLP)."""
    w1, w3, w2, ws1, ws3, ws2 = w
    e0, e1 = expert_block(cfg.n_routed, world_size, rank)
    align = 8 if cfg.dtype == "bf16" else 4
    f0, f1 = shared_block(cfg.shared_inter, world_size, rank, align)
    local = [w1[e0:e1].contiguous(), w3[e0:e1].contiguous(), w2[e0:e1].contiguous()]
    if ws1 is None or f1 == f0:
        return tuple(local) + (None, None, None)
    return tuple(local) + (ws1[f0:f1].contiguous(), ws3[f0:f1].contiguous(),
                           ws2[:, f0:f1].contiguous())


def reduce_partial(y_partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' fp32 shares of y in place (the layer's all_reduce)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial


class EPLayer:
    """One rank of an expert-parallel layer: its weights, workspace and the
    fp32 share buffer. forward() runs the rank's share, the all_reduce and
    the cast."""

    def __init__(self, cfg, T: int, w, world_size: int, rank: int, device, group=None):
        from . import binding as M
        self.M, self.cfg, self.group = M, cfg, group
        self.world_size, self.rank = world_size, rank
        self.begin, self.end = expert_block(cfg.n_routed, world_size, rank)
        self.w = local_weights(cfg, w, world_size, rank)
        self.shared_local = 0 if self.w[3] is None else self.w[3].shape[0]
        self.ws = M.alloc_workspace(cfg, T, device)
        self.y32 = torch.empty(T, cfg.dim, dtype=torch.float32, device=device)

    def partial(self, x, w_r, bias, idx_out: Optional[torch.Tensor] = None, stream=None):
        """This rank's fp32 share of y (before the all_reduce)."""
        self.M.moe_forward_ep(self.cfg, self.begin, self.end, self.shared_local, x, w_r, bias,
                              *self.w, self.y32, self.ws, idx_out=idx_out, stream=stream)
        return self.y32

    def forward(self, x, w_r, bias, y, stream=None) -> None:
        """y = act(sum over ranks of their shares), on `stream` (default: the
        current stream); the all_reduce is issued on the same stream."""
        stream = torch.cuda.current_stream() if stream is None else stream
        self.partial(x, w_r, bias, stream=stream)
        with torch.cuda.stream(stream):
            reduce_partial(self.y32, self.group)
        self.M.moe_cast_output(self.cfg, self.y32, y, stream=stream)
