"""Python-side owner of a libmoe layer and of its pinned host expert store.

``MoELayer`` keeps the pinned host memory that the C library borrows (the
expert set lives in pinned host RAM; the GPU holds a resident copy or a cache
of it) and turns torch tensors into the raw pointers of the C ABI.  All layer
arithmetic runs in libmoe.so.
"""
from __future__ import annotations

import concurrent.futures as cf
from typing import Callable, Optional

import numpy as np
import torch

from . import moe, synth


class MoELayer:
    def __init__(self, hidden: int, inter: int, n_experts: int, top_k: int, n_shared: int,
                 quants=(moe.MOE_Q4_K, moe.MOE_Q4_K, moe.MOE_Q4_K)):
        """quants: GGUF block types of gate, up and down (gate and up share one)."""
        self.H, self.I, self.E, self.k, self.S = hidden, inter, n_experts, top_k, n_shared
        if quants[0] != quants[1]:
            raise ValueError("gate and up weights share one block type")
        self.quants = tuple(quants)
        self.handle = moe.moe_layer_create_mixed(hidden, inter, n_experts, top_k, n_shared, quants[0], quants[2])
        self.gate_bytes = inter * synth.row_bytes(quants[0], hidden)
        self.down_bytes = hidden * synth.row_bytes(quants[2], inter)
        self.expert_bytes = 2 * self.gate_bytes + self.down_bytes   # host (GGUF) bytes
        self.host: Optional[torch.Tensor] = None

    # ------------------------------------------------------------ setup
    def set_router(self, W: np.ndarray, b: Optional[np.ndarray], gating: int) -> None:
        W = np.ascontiguousarray(W, dtype=np.float32)
        bb = None if b is None else np.ascontiguousarray(b, dtype=np.float32)
        moe.moe_set_router(self.handle, W.ctypes.data, None if bb is None else bb.ctypes.data, gating)

    def alloc_host(self) -> torch.Tensor:
        n = self.E + self.S
        self.host = torch.empty(n * self.expert_bytes, dtype=torch.uint8).pin_memory()
        return self.host

    def expert_views(self, e: int):
        """numpy views (gate, up, down) of expert e inside the pinned store."""
        a = self.host.numpy()
        base = e * self.expert_bytes
        g = a[base: base + self.gate_bytes].reshape(self.I, -1)
        u = a[base + self.gate_bytes: base + 2 * self.gate_bytes].reshape(self.I, -1)
        d = a[base + 2 * self.gate_bytes: base + self.expert_bytes].reshape(self.H, -1)
        return g, u, d

    def fill_experts(self, fill: Callable[[int, tuple], None], threads: int = 8) -> None:
        """Call fill(e, (gate, up, down) views) for every expert, in parallel."""
        if self.host is None:
            self.alloc_host()
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda e: fill(e, self.expert_views(e)), range(self.E + self.S)))

    def register_experts(self) -> None:
        n = self.E + self.S
        base = self.host.data_ptr()
        g = [base + e * self.expert_bytes for e in range(n)]
        u = [p + self.gate_bytes for p in g]
        d = [p + 2 * self.gate_bytes for p in g]
        moe.moe_set_experts(self.handle, g, u, d)

    # ------------------------------------------------------------ run
    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        moe.moe_forward(self.handle, x.data_ptr(), out.data_ptr(), T, s)
        return out

    def forward_routed(self, x: torch.Tensor, ids: np.ndarray, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
        T = x.shape[0]
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        if out is None:
            out = torch.empty((T, self.H), dtype=torch.bfloat16, device=x.device)
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        moe.moe_forward_routed(self.handle, x.data_ptr(), out.data_ptr(), T, ids.ctypes.data, s)
        return out

    def routing(self, T: int):
        ids = torch.empty((T, self.k), dtype=torch.int32, device="cuda")
        w = torch.empty((T, self.k), dtype=torch.float32, device="cuda")
        moe.moe_get_routing(self.handle, ids.data_ptr(), w.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return ids, w

    def logits(self, T: int) -> torch.Tensor:
        l = torch.empty((T, self.E), dtype=torch.float32, device="cuda")
        moe.moe_get_logits(self.handle, l.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return l

    def set_expert_parallel(self, rank: int, world: int) -> None:
        moe.moe_set_expert_parallel(self.handle, rank, world)

    def forward_partial(self, x: torch.Tensor, partial: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """This rank's unrounded fp32 share of the output (expert parallelism)."""
        T = x.shape[0]
        if partial is None:
            partial = torch.empty((T, self.H), dtype=torch.float32, device=x.device)
        s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
        moe.moe_forward_partial(self.handle, x.data_ptr(), partial.data_ptr(), T, s)
        return partial

    def prefetch(self, ids) -> None:
        ids = np.ascontiguousarray(ids, dtype=np.int32)
        moe.moe_prefetch(self.handle, ids.ctypes.data, len(ids))

    def destroy(self) -> None:
        if self.handle:
            moe.moe_layer_destroy(self.handle)
            self.handle = 0


def layer_from_config(cfg: synth.LayerConfig, layer_index: int = 0, threads: int = 8) -> MoELayer:
    """Create a layer, fill its pinned store from the seeded generators and
    register router + experts."""
    L = MoELayer(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k, cfg.n_shared, cfg.quants)
    L.set_router(synth.router_weight(cfg, layer_index), synth.router_bias(cfg, layer_index), cfg.gating)

    def fill(e, views):
        for m, v in enumerate(views):
            rows, cols = (cfg.inter, cfg.hidden) if m < 2 else (cfg.hidden, cfg.inter)
            synth.q_tensor(cfg.quants[m], cfg.seed, layer_index, e, m, rows, cols, out=v)

    L.fill_experts(fill, threads)
    L.register_experts()
    return L
