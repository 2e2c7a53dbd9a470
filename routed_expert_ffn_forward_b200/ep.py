"""Expert parallelism across GPUs, one rank (process) per GPU.

Each rank's layer owns the experts e with e % world == rank
(``moe_set_expert_parallel``), so it holds, caches and streams only those.
A forward is three steps:

1. ``moe_forward_partial``: every rank runs the whole router, then only its
   own experts, and sums their weighted outputs per token in the fixed combine
   order -- an unrounded fp32 partial [T, H];
2. one all-gather of the partials over NCCL (T*H*4 bytes per rank), which
   leaves them stacked in rank order on every rank;
3. ``moe_combine_partials``: the partials added in rank order and rounded to
   bf16 once, so every rank ends with the same bits on every run (LayerStoRm
   README, "Notes": expert parallelism with a deterministic combine).

The all-gather is the library collective; the arithmetic of steps 1 and 3
runs in libmoe.so.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import moe


def exchange(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Every rank's `partial`, stacked in rank order: [world, *partial.shape]."""
    world = dist.get_world_size(group)
    p = partial.contiguous()
    flat = torch.empty((world * p.shape[0],) + tuple(p.shape[1:]), dtype=p.dtype, device=p.device)
    dist.all_gather_into_tensor(flat, p, group=group)     # rank r's rows land at r * rows
    return flat.view((world,) + tuple(p.shape))


def ep_forward(layer, x: torch.Tensor, group=None, stream=None) -> torch.Tensor:
    """The layer's output on this rank, computed with expert parallelism
    (the layer must have been given this rank and the world size)."""
    T, H = x.shape[0], layer.H
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    partial = layer.forward_partial(x, stream=s)
    gathered = exchange(partial, group)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    moe.moe_combine_partials(gathered.data_ptr(), out.data_ptr(), T, H, gathered.shape[0], s)
    return out
