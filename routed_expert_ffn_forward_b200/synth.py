"""Seeded synthetic inputs for the routed-expert FFN layer.

This module only *draws* inputs: activations, router weights and bias, Q4_K
expert tensors and the expert-streaming routing trace.  It holds none of the
layer's arithmetic (no dequantisation, no routing, no FFN), so the CPU oracle
and the CUDA path can both consume its output without sharing any of the
method's code.

Every tensor comes from its own counter-based stream: numpy's Philox keyed by
``(seed, stream id)``, where the stream id packs what the tensor is and where it
sits (layer, expert, matrix).  Any single expert can therefore be regenerated on
demand without drawing the rest of the model, which is what lets the oracle
check a sampled expert of a 51 GB stacked model.

Workload shapes follow the pages' model family (LayerStoRm README, "References":
a DeepSeek-V3-style MLA + MoE model served from GGUF UD-Q4_K_XL weights): hidden
7168, expert inter 2048, 256 routed experts, top-8, one shared expert.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Q4_K super-block: 256 weights in 144 bytes (fp16 d, fp16 dmin, 12 bytes of
# packed 6-bit scales/mins, 128 bytes of 4-bit quants).  Public GGUF format.
QK_K = 256
Q4K_BLOCK_BYTES = 144

# GGUF block types (GGML type id -> (weights per block, bytes per block))
Q8_0, Q4_K, Q5_K, Q6_K, MXFP4 = 8, 12, 13, 14, 39
BLOCKS = {Q8_0: (32, 34), Q4_K: (256, 144), Q5_K: (256, 176), Q6_K: (256, 210), MXFP4: (32, 17)}


def row_bytes(qtype: int, cols: int) -> int:
    """Bytes of one weight row of `cols` inputs (padded to whole blocks)."""
    n, b = BLOCKS[qtype]
    return (cols + n - 1) // n * b


GATE, UP, DOWN = 0, 1, 2

# stream kinds (high byte of the Philox stream id)
_K_WEIGHT, _K_X, _K_ROUTER, _K_BIAS, _K_TRACE = 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape and distribution parameters of one synthetic MoE layer workload."""

    name: str
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    n_shared: int
    tokens: int
    gating: int            # 0 = softmax over the top-k logits, 1 = sigmoid + renormalise
    seed: int
    router_std: float      # router weight ~ N(0, router_std^2)
    zipf_s: Optional[float] = None   # router bias -s*ln(rank); None = zero bias
    n_layers: int = 1
    cache_bytes: Optional[int] = None
    steps: int = 1
    keep_p: float = 0.6
    quants: tuple = (Q4_K, Q4_K, Q4_K)    # GGUF block types of gate, up, down

    @property
    def blocks_h(self) -> int:
        return (self.hidden + QK_K - 1) // QK_K

    @property
    def blocks_i(self) -> int:
        return (self.inter + QK_K - 1) // QK_K

    @property
    def gate_bytes(self) -> int:
        return self.inter * row_bytes(self.quants[0], self.hidden)

    @property
    def up_bytes(self) -> int:
        return self.inter * row_bytes(self.quants[1], self.hidden)

    @property
    def down_bytes(self) -> int:
        return self.hidden * row_bytes(self.quants[2], self.inter)

    @property
    def expert_bytes(self) -> int:
        return self.gate_bytes + self.up_bytes + self.down_bytes


H, I = 7168, 2048
TINY = LayerConfig("tiny: H=256 I=128 E=16 k=2 S=0 T=4 softmax", 256, 128, 16, 2, 0, 4,
                   0, 0, 1.0 / 16.0)
DECODE = LayerConfig("decode: H=7168 I=2048 E=256+1 k=8 T=1 sigmoid, resident", H, I, 256, 8, 1, 1,
                     1, 1, 1.0 / math.sqrt(H))
BATCHED = LayerConfig("batched decode: T=64, Zipf(1.1) router bias", H, I, 256, 8, 1, 64,
                      1, 2, 1.0 / math.sqrt(H), zipf_s=1.1)
PREFILL = LayerConfig("prefill chunk: T=4096, Zipf(0.8) router bias", H, I, 256, 8, 1, 4096,
                      1, 3, 1.0 / math.sqrt(H), zipf_s=0.8)
STREAMING = LayerConfig("expert streaming: 8 layers, 12e9 B cache, T=1, 512 steps", H, I, 256, 8, 1, 1,
                        1, 4, 1.0 / math.sqrt(H), n_layers=8, cache_bytes=12_000_000_000, steps=512,
                        zipf_s=1.1)
# bench.py --config N selects WORKLOADS[N]
WORKLOADS = {0: TINY, 1: DECODE, 2: BATCHED, 3: PREFILL, 4: STREAMING}


def _gen(seed: int, kind: int, a: int = 0, b: int = 0, c: int = 0) -> np.random.Generator:
    sid = (kind << 56) | ((a & 0xFFFFFF) << 32) | ((b & 0xFFFFFF) << 8) | (c & 0xFF)
    return np.random.Generator(np.random.Philox(key=np.array([seed, sid], dtype=np.uint64)))


def round_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float array -> bf16 bit patterns (uint16), via fp32 then round-to-nearest-even.

    Used only to *draw* bf16 activations; the oracle rounds its outputs with its
    own routine.
    """
    f = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (f + 0x7FFF + ((f >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def q4k_tensor(seed: int, layer: int, expert: int, matrix: int, rows: int, cols: int,
               out: Optional[np.ndarray] = None) -> np.ndarray:
    """Draw one Q4_K weight matrix [rows, cols] as raw bytes [rows, nb*144].

    Rows hold ceil(cols/256) consecutive super-blocks along the input dimension.
    d ~ U(1e-3, 1e-2) and dmin ~ U(0, 5e-3) are drawn in fp64 and rounded to
    fp16 (RNE); the 12 scale bytes and 128 quant bytes are uniform random bytes,
    which makes every 6-bit scale/min uniform on 0..63 and every quant uniform
    on 0..15 (the 12-byte packing is a bijection of 96 bits onto 16 six-bit
    fields).
    """
    nb = (cols + QK_K - 1) // QK_K
    n = rows * nb
    g = _gen(seed, _K_WEIGHT, layer, expert, matrix)
    d = g.uniform(1e-3, 1e-2, n).astype(np.float16)
    dmin = g.uniform(0.0, 5e-3, n).astype(np.float16)
    if out is None:
        out = np.empty((rows, nb * Q4K_BLOCK_BYTES), dtype=np.uint8)
    blk = out.reshape(n, Q4K_BLOCK_BYTES)
    blk[:, 4:] = g.integers(0, 256, size=(n, Q4K_BLOCK_BYTES - 4), dtype=np.uint8)
    blk[:, 0:2] = d.view(np.uint8).reshape(n, 2)
    blk[:, 2:4] = dmin.view(np.uint8).reshape(n, 2)
    return out


def q_tensor(qtype: int, seed: int, layer: int, expert: int, matrix: int, rows: int, cols: int,
             out: Optional[np.ndarray] = None) -> np.ndarray:
    """Draw one weight matrix [rows, cols] of any supported GGUF block type as
    raw bytes [rows, row_bytes].  Quant bytes are uniform random; the scale
    fields are drawn so that weights are of order one, like the Q4_K ones:
      Q4_K  d ~ U(1e-3, 1e-2), dmin ~ U(0, 5e-3)             (q4k_tensor)
      Q5_K  d ~ U(5e-4, 5e-3), dmin ~ U(0, 5e-3)             (q up to 31)
      Q6_K  d ~ U(5e-5, 5e-4), 16 int8 scales uniform        (|w| <= d*128*32)
      Q8_0  d ~ U(1e-3, 1e-2)                                (|w| <= d*128)
      MXFP4 scale exponent e uniform on 124..127             (|w| <= 6)
    fp16 fields are drawn in fp64 and rounded to fp16."""
    if qtype == Q4_K:
        return q4k_tensor(seed, layer, expert, matrix, rows, cols, out)
    n_el, nbytes = BLOCKS[qtype]
    nb = (cols + n_el - 1) // n_el
    n = rows * nb
    g = _gen(seed, _K_WEIGHT, layer, expert, matrix)
    if out is None:
        out = np.empty((rows, nb * nbytes), dtype=np.uint8)
    blk = out.reshape(n, nbytes)
    blk[:] = g.integers(0, 256, size=(n, nbytes), dtype=np.uint8)
    f16 = lambda v: v.astype(np.float16).view(np.uint8).reshape(n, 2)
    if qtype == Q5_K:
        blk[:, 0:2] = f16(g.uniform(5e-4, 5e-3, n))
        blk[:, 2:4] = f16(g.uniform(0.0, 5e-3, n))
    elif qtype == Q6_K:
        blk[:, 208:210] = f16(g.uniform(5e-5, 5e-4, n))
    elif qtype == Q8_0:
        blk[:, 0:2] = f16(g.uniform(1e-3, 1e-2, n))
    elif qtype == MXFP4:
        blk[:, 0] = g.integers(124, 128, size=n, dtype=np.uint8)
    return out


def expert_tensors(cfg: LayerConfig, layer: int, expert: int):
    """(gate, up, down) raw bytes of the configured block types for routed
    expert ``expert`` (shared experts are numbered E..E+S-1)."""
    qg, qu, qd = cfg.quants
    gate = q_tensor(qg, cfg.seed, layer, expert, GATE, cfg.inter, cfg.hidden)
    up = q_tensor(qu, cfg.seed, layer, expert, UP, cfg.inter, cfg.hidden)
    down = q_tensor(qd, cfg.seed, layer, expert, DOWN, cfg.hidden, cfg.inter)
    return gate, up, down


def activations(cfg: LayerConfig, layer: int = 0, step: int = 0, tokens: Optional[int] = None) -> np.ndarray:
    """x ~ N(0,1) rounded to bf16, as uint16 bits [T, H]."""
    t = cfg.tokens if tokens is None else tokens
    g = _gen(cfg.seed, _K_X, layer, step)
    return round_bf16_bits(g.standard_normal((t, cfg.hidden)))


def router_weight(cfg: LayerConfig, layer: int = 0) -> np.ndarray:
    """Router weight fp32 [E, H] ~ N(0, router_std^2)."""
    g = _gen(cfg.seed, _K_ROUTER, layer)
    return (g.standard_normal((cfg.n_experts, cfg.hidden)) * cfg.router_std).astype(np.float32)


def router_bias(cfg: LayerConfig, layer: int = 0) -> np.ndarray:
    """Router bias fp32 [E].  Zero, or -s*ln(r_e) with r a seeded permutation of
    1..E so that expert popularity falls off like a Zipf(s) law."""
    if cfg.zipf_s is None:
        return np.zeros(cfg.n_experts, dtype=np.float32)
    g = _gen(cfg.seed, _K_BIAS, layer)
    r = g.permutation(cfg.n_experts) + 1
    return (-cfg.zipf_s * np.log(r.astype(np.float64))).astype(np.float32)


def streaming_trace(cfg: LayerConfig) -> np.ndarray:
    """Temporally correlated routing trace int32 [steps, layers, top_k].

    Per layer, experts get a seeded popularity rank and are drawn by Zipf(s)
    over rank.  Step 0 draws top_k distinct experts; every later step keeps each
    previous expert with probability keep_p and refills the rest by Zipf draws,
    rejecting duplicates.  Kept experts come first, in their previous order.
    """
    E, k, s = cfg.n_experts, cfg.top_k, cfg.zipf_s or 1.1
    out = np.empty((cfg.steps, cfg.n_layers, k), dtype=np.int32)
    p = 1.0 / np.arange(1, E + 1, dtype=np.float64) ** s
    p /= p.sum()
    for layer in range(cfg.n_layers):
        g = _gen(cfg.seed, _K_TRACE, layer)
        rank_to_expert = g.permutation(E)
        prev: list[int] = []
        for step in range(cfg.steps):
            cur = [e for e in prev if g.random() < cfg.keep_p] if step else []
            while len(cur) < k:
                e = int(rank_to_expert[g.choice(E, p=p)])
                if e not in cur:
                    cur.append(e)
            out[step, layer] = cur
            prev = cur
    return out


def pinned_workload_bytes(cfg: LayerConfig) -> int:
    return cfg.n_layers * (cfg.n_experts + cfg.n_shared) * cfg.expert_bytes
