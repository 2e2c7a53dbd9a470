"""CPU oracle for the routed mixture-of-experts FFN layer (numpy, fp64).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module:
only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA path; its inputs come from the seeded generators in
``routed_expert_ffn_forward_b200.synth``, which hold none of the layer's
arithmetic.

What it computes (sparse routing reaches the dense definition exactly, so the
oracle is that definition written out, step by step, slowly and plainly):

1. router logits  l[t,e] = sum_h x[t,h] * Wr[e,h] + b[e]              (fp64)
2. top-k          S_t = the k largest logits, ties to the lower expert index
3. gate weights   softmax over l[t,S_t] (gating 0) or
                  sigmoid(l[t,S_t]) / sum sigmoid(l[t,S_t]) (gating 1)
4. expert FFN     h = silu(W_g x) * (W_u x),  y = W_d h,  W dequantised from Q4_K
5. combine        out[t] = sum_j w[t,j] * y_(S_t[j]) + sum_s y_(shared s)
6. output         out rounded to bf16, round-to-nearest-even

Sources.  The pages (LayerStoRm README, "TL;DR": each token activates only a
few experts chosen by the router; "Get a model": GGUF UD-Q4_K_XL weights;
"References": the DeepSeek-V3 MLA + MoE architecture; "Notes": a deterministic
expert-parallel combine) describe the layer in prose only.  They define neither
Q4_K, the gating function nor SwiGLU, so:

* Q4_K follows the public GGUF k-quant super-block layout (see ``q4k_dequant``).
* gating, bias handling and SwiGLU take the plainest reading: the bias is added
  to the logits and used for both selection and weights; no group-limited
  routing; routed scaling factor 1; the shared expert is always on with weight
  1; silu is applied to the gate projection.
* An inter size that is not a multiple of 256 is padded to whole super-blocks
  along the down projection's input; the padded inputs of h are zero, so those
  weights contribute exactly nothing.

Every function here is pinned by ``tests/test_oracle.py`` against something
other than itself (a hand-worked block, the ``gguf`` library, closed forms,
library routines and a brute-force dense MoE).
"""
from __future__ import annotations

import numpy as np

QK_K = 256
BLOCK_BYTES = 144


# --------------------------------------------------------------------------- Q4_K
def q4k_scale_min(scales: np.ndarray):
    """Unpack the 12 scale bytes of each super-block into 8 six-bit scales and
    8 six-bit mins (GGUF k-quant layout).

    Sub-blocks 0..3 keep their scale and min in the low 6 bits of bytes j and
    j+4.  Sub-blocks 4..7 take their low 4 bits from the nibbles of byte j+4
    (scale: low nibble, min: high nibble) and their top 2 bits from the spare
    top bits of bytes j-4 (scale) and j (min).
    """
    s = scales.astype(np.int64)
    sc = np.empty(s.shape[:-1] + (8,), dtype=np.int64)
    mn = np.empty_like(sc)
    for j in range(4):
        sc[..., j] = s[..., j] & 63
        mn[..., j] = s[..., j + 4] & 63
    for j in range(4, 8):
        sc[..., j] = (s[..., j + 4] & 0x0F) | ((s[..., j - 4] >> 6) << 4)
        mn[..., j] = (s[..., j + 4] >> 4) | ((s[..., j] >> 6) << 4)
    return sc, mn


def q4k_dequant(raw: np.ndarray) -> np.ndarray:
    """Dequantise Q4_K bytes [..., nb*144] to fp64 weights [..., nb*256], exactly.

    One 144-byte super-block holds 256 weights in 8 sub-blocks of 32:
      bytes 0-1   d    (fp16)    super-block scale
      bytes 2-3   dmin (fp16)    super-block min scale
      bytes 4-15  packed 6-bit scale sc_j and min m_j of sub-block j
      bytes 16-143 quants: four chunks of 32 bytes; in chunk c, the low nibble
                  of byte i is weight 64c+i (sub-block 2c) and the high nibble
                  is weight 64c+32+i (sub-block 2c+1)
    weight = d*sc_j*q - dmin*m_j.  Products of an fp16 and small integers are
    exact in fp64, so the result is the exact value of the format.
    """
    raw = np.asarray(raw, dtype=np.uint8)
    lead = raw.shape[:-1]
    nb = raw.shape[-1] // BLOCK_BYTES
    b = raw.reshape(lead + (nb, BLOCK_BYTES))
    d = b[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    dmin = b[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    sc, mn = q4k_scale_min(b[..., 4:16])
    qs = b[..., 16:144].reshape(lead + (nb, 4, 32)).astype(np.int64)
    q = np.empty(lead + (nb, 8, 32), dtype=np.int64)
    q[..., 0::2, :] = qs & 0x0F          # sub-block 2c: low nibbles of chunk c
    q[..., 1::2, :] = qs >> 4            # sub-block 2c+1: high nibbles of chunk c
    w = d[..., None, None] * sc[..., None] * q - dmin[..., None, None] * mn[..., None]
    return w.reshape(lead + (nb * QK_K,))


# --------------------------------------------------------------------------- other GGUF block types
# UD-Q*_K_XL files mix block types per tensor (LayerStoRm README, "Get a
# model"; "License and attributions": GGUF and MXFP4 decode paths).  Each
# function below dequantises one public GGUF block type exactly, in fp64.
# GGML type ids: Q8_0 = 8, Q4_K = 12, Q5_K = 13, Q6_K = 14, MXFP4 = 39.

Q8_0, Q4_K, Q5_K, Q6_K, MXFP4 = 8, 12, 13, 14, 39
BLOCK = {Q8_0: (32, 34), Q4_K: (256, 144), Q5_K: (256, 176), Q6_K: (256, 210), MXFP4: (32, 17)}


def _blocks(raw, nbytes):
    raw = np.asarray(raw, dtype=np.uint8)
    lead = raw.shape[:-1]
    nb = raw.shape[-1] // nbytes
    return raw.reshape(lead + (nb, nbytes)), lead, nb


def _f16(two_bytes):
    return two_bytes.copy().view(np.float16)[..., 0].astype(np.float64)


def q8_0_dequant(raw):
    """Q8_0: blocks of 32 weights in 34 bytes: fp16 d, then 32 signed bytes q;
    weight = d * q."""
    b, lead, nb = _blocks(raw, 34)
    d = _f16(b[..., 0:2])
    q = b[..., 2:34].view(np.int8).astype(np.float64)
    return (d[..., None] * q).reshape(lead + (nb * 32,))


def q5_k_dequant(raw):
    """Q5_K: 256 weights in 176 bytes: fp16 d, fp16 dmin, the 12 packed scale
    bytes of Q4_K (eight 6-bit scales and mins), 32 bytes of fifth bits qh,
    128 bytes of low nibbles qs.  Chunk c (64 weights) takes bytes 32c..32c+31
    of qs: the low nibble of byte i is weight 64c+i (sub-block 2c, fifth bit =
    bit 2c of qh[i]), the high nibble weight 64c+32+i (sub-block 2c+1, fifth
    bit = bit 2c+1 of qh[i]).  weight = d*sc_j*q - dmin*m_j, q in 0..31."""
    b, lead, nb = _blocks(raw, 176)
    d, dmin = _f16(b[..., 0:2]), _f16(b[..., 2:4])
    sc, mn = q4k_scale_min(b[..., 4:16])
    qh = b[..., 16:48].astype(np.int64)
    qs = b[..., 48:176].reshape(lead + (nb, 4, 32)).astype(np.int64)
    q = np.empty(lead + (nb, 8, 32), dtype=np.int64)
    for c in range(4):
        q[..., 2 * c, :] = (qs[..., c, :] & 0x0F) | (((qh >> (2 * c)) & 1) << 4)
        q[..., 2 * c + 1, :] = (qs[..., c, :] >> 4) | (((qh >> (2 * c + 1)) & 1) << 4)
    w = d[..., None, None] * sc[..., None] * q - dmin[..., None, None] * mn[..., None]
    return w.reshape(lead + (nb * 256,))


def q6_k_dequant(raw):
    """Q6_K: 256 weights in 210 bytes: 128 bytes of low nibbles ql, 64 bytes of
    high bit pairs qh, 16 signed 8-bit scales, fp16 d.  Two halves of 128
    weights, half h using ql[64h..], qh[32h..], scales[8h..].  Within a half,
    for i in 0..31 and g = i // 16, the four weights
      i      : low nibble of ql[i],      bits 0-1 of qh[i], scale g
      i + 32 : low nibble of ql[i + 32], bits 2-3 of qh[i], scale g + 2
      i + 64 : high nibble of ql[i],     bits 4-5 of qh[i], scale g + 4
      i + 96 : high nibble of ql[i + 32], bits 6-7 of qh[i], scale g + 6
    have the 6-bit value q = nibble | (pair << 4); weight = d * scale * (q - 32)."""
    b, lead, nb = _blocks(raw, 210)
    ql = b[..., 0:128].astype(np.int64)
    qh = b[..., 128:192].astype(np.int64)
    scales = b[..., 192:208].view(np.int8).astype(np.float64)
    d = _f16(b[..., 208:210])
    w = np.empty(lead + (nb, 256), dtype=np.float64)
    for h in range(2):
        L, Hh, S = ql[..., 64 * h:64 * h + 64], qh[..., 32 * h:32 * h + 32], scales[..., 8 * h:8 * h + 8]
        for part, (lo, sh, nib_hi, off) in enumerate(((0, 0, False, 0), (32, 2, False, 2),
                                                       (0, 4, True, 4), (32, 6, True, 6))):
            nib = (L[..., lo:lo + 32] >> 4) if nib_hi else (L[..., lo:lo + 32] & 0x0F)
            q = (nib | (((Hh >> sh) & 3) << 4)) - 32
            g = np.arange(32) // 16
            sc = S[..., off + g]
            w[..., 128 * h + 32 * part:128 * h + 32 * part + 32] = d[..., None] * sc * q
    return w.reshape(lead + (nb * 256,))


# FP4 E2M1 values of the 16 codes (bit 3 = sign): 0, 0.5, 1, 1.5, 2, 3, 4, 6
_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def mxfp4_dequant(raw):
    """MXFP4 (OCP microscaling FP4): blocks of 32 weights in 17 bytes: an E8M0
    scale byte e (the power of two 2^(e-127)), then 16 bytes of FP4 E2M1 codes:
    element i is the low nibble of byte i, element 16+i its high nibble;
    weight = e2m1(code) * 2^(e-127)."""
    b, lead, nb = _blocks(raw, 17)
    e = b[..., 0].astype(np.int64)
    qs = b[..., 1:17].astype(np.int64)
    codes = np.concatenate([qs & 0x0F, qs >> 4], axis=-1)
    w = _E2M1[codes] * np.ldexp(1.0, e - 127)[..., None]
    return w.reshape(lead + (nb * 32,))


def dequant(raw, qtype: int) -> np.ndarray:
    """Dequantise a matrix of any supported GGUF block type ([..., row bytes])."""
    fn = {Q4_K: q4k_dequant, Q5_K: q5_k_dequant, Q6_K: q6_k_dequant, Q8_0: q8_0_dequant,
          MXFP4: mxfp4_dequant}[qtype]
    return fn(raw)


# --------------------------------------------------------------------------- router
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp64, exactly."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def router_logits(x: np.ndarray, w_router: np.ndarray, bias) -> np.ndarray:
    """l[t,e] = sum_h x[t,h] Wr[e,h] + b[e] in fp64 (x, Wr exact in fp64)."""
    l = np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T
    if bias is not None:
        l = l + np.asarray(bias, np.float64)[None, :]
    return l


def topk_ids(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest logits per row, largest first; equal logits go
    to the lower expert index."""
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-logits[t, e], e))
        ids[t] = order[:k]
    return ids


def gate_weights(logits: np.ndarray, ids: np.ndarray, gating: int) -> np.ndarray:
    """Weights of the selected experts.

    gating 0: softmax over the k selected logits.
    gating 1: sigmoid of each selected logit, renormalised to sum 1.
    """
    sel = np.take_along_axis(logits, ids, axis=1)
    if gating == 0:
        z = np.exp(sel - sel.max(axis=1, keepdims=True))
        return z / z.sum(axis=1, keepdims=True)
    sig = 1.0 / (1.0 + np.exp(-sel))
    return sig / sig.sum(axis=1, keepdims=True)


def route(x, w_router, bias, k: int, gating: int):
    """Router step: (ids [T,k], weights [T,k], logits [T,E])."""
    l = router_logits(x, w_router, bias)
    ids = topk_ids(l, k)
    return ids, gate_weights(l, ids, gating), l


def topk_gap(logits: np.ndarray, k: int) -> np.ndarray:
    """l_(k) - l_(k+1) per token (k-th minus (k+1)-th largest logit); +inf if k == E."""
    s = -np.sort(-logits, axis=1)
    if k >= logits.shape[1]:
        return np.full(logits.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


# --------------------------------------------------------------------------- permutation
def permutation(ids: np.ndarray, n_experts: int):
    """Counting-sort permutation of the (token, slot) pairs by expert.

    counts[e] = #{(t,j): ids[t,j] = e}; offsets = exclusive prefix sum;
    perm lists flat pair indices t*k+j ordered by (e, t, j).
    """
    T, k = ids.shape
    counts = np.zeros(n_experts, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[ids[t, j]] += 1
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    for e in range(n_experts):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:-1].copy()
    perm = np.empty(T * k, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = ids[t, j]
            perm[fill[e]] = t * k + j
            fill[e] += 1
    return counts, offsets, perm


# --------------------------------------------------------------------------- experts
def silu(z):
    return z / (1.0 + np.exp(-z))


def expert_ffn(xr: np.ndarray, gate_raw, up_raw, down_raw, inter: int, quants=(Q4_K, Q4_K, Q4_K)) -> np.ndarray:
    """SwiGLU expert on rows xr [n, H] (fp64): y = W_d (silu(W_g x) * (W_u x));
    `quants` are the GGUF block types of gate, up and down."""
    wg = dequant(gate_raw, quants[0])             # [I, H]
    wu = dequant(up_raw, quants[1])               # [I, H]
    wd = dequant(down_raw, quants[2])             # [H, I_pad]
    h = silu(xr @ wg.T) * (xr @ wu.T)             # [n, I]
    return h @ wd[:, :inter].T                    # padded inputs of h are zero


def round_bf16(v: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 (ties to even), returned as uint16 bit patterns.

    Exact: works on the fp64 value itself (no fp32 detour), by locating the
    bf16 grid spacing around |v| and rounding on that grid.
    """
    v = np.asarray(v, np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    flat, res = v.ravel(), out.ravel()
    for i, a in enumerate(flat):
        if a == 0.0:
            res[i] = 0x8000 if np.signbit(a) else 0
            continue
        m, e = np.frexp(abs(a))                 # |a| = m * 2^e, m in [0.5, 1)
        e = max(e, -125)                        # subnormal bf16 share one spacing
        ulp = np.ldexp(1.0, e - 8)              # 8 significant bits
        q = abs(a) / ulp
        r = np.floor(q)
        if q - r > 0.5 or (q - r == 0.5 and int(r) % 2 == 1):
            r += 1
        f = np.float32(np.copysign(r * ulp, a))  # representable in fp32 exactly
        res[i] = (np.array(f, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    return out


def moe_forward(x_bits: np.ndarray, layer, k: int, gating: int, n_shared: int,
                inter: int, forced_ids=None, token_subset=None):
    """Whole layer on the CPU.

    layer: dict with 'router_w' [E,H] fp32, 'router_b' [E] or None,
           'experts': callable e -> (gate_raw, up_raw, down_raw) for
           e in 0..E+S-1 (shared experts numbered after the routed ones) and
           optionally 'quants': the GGUF block types of gate, up and down
           (default Q4_K for all three).
    forced_ids: optional [T,k] expert ids to use instead of the top-k (the
           weights are then the gating function of the logits at those ids).
    token_subset: optional token indices; only those output rows are computed.
    Returns dict(out64 [n,H], out_bf16 [n,H] uint16, ids, w, logits, gap, tokens).
    """
    x = bf16_to_f64(x_bits)
    tokens = np.arange(x.shape[0]) if token_subset is None else np.asarray(token_subset)
    xs = x[tokens]
    l = router_logits(xs, layer["router_w"], layer.get("router_b"))
    E = l.shape[1]
    if forced_ids is None:
        ids = topk_ids(l, k)
    else:
        ids = np.asarray(forced_ids, dtype=np.int64)[tokens]
    w = gate_weights(l, ids, gating)
    out = np.zeros((len(tokens), x.shape[1]), dtype=np.float64)
    needed = sorted(set(int(e) for e in ids.ravel()))
    for e in needed:
        rows = [(n, j) for n in range(len(tokens)) for j in range(k) if ids[n, j] == e]
        ns = [n for n, _ in rows]
        y = expert_ffn(xs[ns], *layer["experts"](e), inter, layer.get("quants", (Q4_K,) * 3))
        for (n, j), yr in zip(rows, y):
            out[n] += w[n, j] * yr
    for s in range(n_shared):
        out += expert_ffn(xs, *layer["experts"](E + s), inter, layer.get("quants", (Q4_K,) * 3))
    return dict(out64=out, out_bf16=round_bf16(out), ids=ids, w=w, logits=l,
                gap=topk_gap(l, k), tokens=tokens)


def dense_moe(x_bits: np.ndarray, layer, k: int, gating: int, n_shared: int, inter: int):
    """Brute force: run EVERY expert on EVERY token, then mask with a dense gate
    vector that is zero outside each token's top-k.  Independent of the sparse
    routing/permutation bookkeeping; used to pin ``moe_forward`` on small shapes."""
    x = bf16_to_f64(x_bits)
    l = router_logits(x, layer["router_w"], layer.get("router_b"))
    T, E = l.shape
    gate = np.zeros((T, E))
    for t in range(T):
        order = np.lexsort((np.arange(E), -l[t]))[:k]
        sel = l[t, order]
        if gating == 0:
            z = np.exp(sel - sel.max())
            gate[t, order] = z / z.sum()
        else:
            sg = 1.0 / (1.0 + np.exp(-sel))
            gate[t, order] = sg / sg.sum()
    out = np.zeros_like(x)
    for e in range(E):
        out += gate[:, e:e + 1] * expert_ffn(x, *layer["experts"](e), inter, layer.get("quants", (Q4_K,) * 3))
    for s in range(n_shared):
        out += expert_ffn(x, *layer["experts"](E + s), inter, layer.get("quants", (Q4_K,) * 3))
    return out
