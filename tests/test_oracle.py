"""Pins for the CPU oracle (CPU only).

Each test checks the oracle against something other than itself: a
hand-worked Q4_K block, the ``gguf`` library's own dequantiser, closed forms,
library routines (numpy's stable argsort, scipy's softmax, torch's bf16 cast)
and a brute-force dense MoE.  ``test_pins_catch_planted_mistakes`` plants
plausible bugs in the oracle and checks that the pins catch every one.
"""
import json
import os

import numpy as np
import pytest

from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ helpers
def pack_scales(sc: np.ndarray, mn: np.ndarray) -> np.ndarray:
    """Inverse of the k-quant scale packing: 8 six-bit (scale, min) pairs -> 12 bytes.
    Written as the packing (not the unpacking) so a round trip pins the oracle."""
    out = np.zeros(sc.shape[:-1] + (12,), dtype=np.int64)
    for j in range(4):
        out[..., j] |= sc[..., j] & 63
        out[..., j + 4] |= mn[..., j] & 63
    for j in range(4, 8):
        out[..., j + 4] |= (sc[..., j] & 15) | ((mn[..., j] & 15) << 4)
        out[..., j - 4] |= (sc[..., j] >> 4) << 6
        out[..., j] |= (mn[..., j] >> 4) << 6
    return out.astype(np.uint8)


def make_block(d, dmin, sc, mn, q):
    """Build one 144-byte block from fields (q: 256 quants in weight order)."""
    b = np.zeros(144, dtype=np.uint8)
    b[0:2] = np.frombuffer(np.float16(d).tobytes(), np.uint8)
    b[2:4] = np.frombuffer(np.float16(dmin).tobytes(), np.uint8)
    b[4:16] = pack_scales(np.asarray(sc)[None], np.asarray(mn)[None])[0]
    q = np.asarray(q, dtype=np.int64).reshape(4, 2, 32)     # chunk, half, i
    b[16:] = (q[:, 0, :] | (q[:, 1, :] << 4)).reshape(128).astype(np.uint8)
    return b


def tiny_layer(cfg, zero_routed=False, const_block=None):
    """Layer dict for the oracle from the seeded generators."""
    cache = {}

    def experts(e):
        if e not in cache:
            g, u, d = synth.expert_tensors(cfg, 0, e)
            if const_block is not None:
                blocks = const_block if isinstance(const_block, tuple) else (const_block,) * 3
                for m, blk in zip((g, u, d), blocks):
                    m.reshape(-1, 144)[:] = blk
            if zero_routed and e < cfg.n_experts:
                for m in (g, u, d):
                    m.reshape(-1, 144)[:, 0:4] = 0          # d = dmin = 0
            cache[e] = (g, u, d)
        return cache[e]

    return dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg), experts=experts)


def cfg_with(base, **kw):
    import dataclasses
    return dataclasses.replace(base, **kw)


# ------------------------------------------------------------------ Q4_K
def test_q4k_hand_block():
    doc = json.load(open(os.path.join(GOLDEN, "q4k_hand_block.json")))
    blk = np.frombuffer(bytes.fromhex(doc["block_hex"]), dtype=np.uint8)
    w = ref.q4k_dequant(blk)
    assert w.shape == (256,)
    np.testing.assert_array_equal(w, np.array(doc["expected"], dtype=np.float64))


def test_q4k_scale_pack_round_trip():
    rng = np.random.default_rng(5)
    sc = rng.integers(0, 64, (500, 8))
    mn = rng.integers(0, 64, (500, 8))
    s2, m2 = ref.q4k_scale_min(pack_scales(sc, mn))
    np.testing.assert_array_equal(s2, sc)
    np.testing.assert_array_equal(m2, mn)


def test_q4k_closed_form_constant():
    # constant q, constant sc, m = 0  =>  every weight is d*sc*q
    blk = make_block(0.0625, 0.5, [5] * 8, [0] * 8, [9] * 256)
    np.testing.assert_array_equal(ref.q4k_dequant(blk), np.full(256, 0.0625 * 5 * 9))
    # q = 0 everywhere => every weight is -dmin*m_j
    mn = [1, 2, 3, 4, 60, 61, 62, 63]
    blk = make_block(0.25, 0.125, [7] * 8, mn, [0] * 256)
    np.testing.assert_array_equal(ref.q4k_dequant(blk), np.repeat(-0.125 * np.array(mn, float), 32))


def test_q4k_weight_order():
    # a single non-zero quant lands at exactly one weight position
    for pos in (0, 31, 32, 63, 64, 100, 191, 255):
        q = np.zeros(256, dtype=np.int64)
        q[pos] = 15
        w = ref.q4k_dequant(make_block(1.0, 0.0, [1] * 8, [0] * 8, q))
        assert np.flatnonzero(w).tolist() == [pos] and w[pos] == 15.0


def test_q4k_matches_gguf_library():
    gguf = pytest.importorskip("gguf")
    from gguf.quants import dequantize
    raw = synth.q4k_tensor(7, 0, 3, 0, 16, 1024)
    ours = ref.q4k_dequant(raw)
    lib = dequantize(raw, gguf.GGMLQuantizationType.Q4_K).astype(np.float64).reshape(ours.shape)
    np.testing.assert_allclose(ours, lib, rtol=2e-6, atol=1e-6)


# ------------------------------------------------------------------ bf16 rounding
def test_round_bf16_matches_torch_on_fp32_values():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(4000) * 10.0 ** rng.integers(-30, 30, 4000),
                        [0.0, -0.0, 1.0, -2.5, 3.3895e38, 1e-39, -1e-40]]).astype(np.float32)
    expect = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ref.round_bf16(v.astype(np.float64)), expect)


def test_round_bf16_ties_and_single_rounding():
    one = 0x3F80
    assert ref.round_bf16(np.array([1.0 + 2 ** -8]))[0] == one               # tie -> even
    assert ref.round_bf16(np.array([1.0 + 3 * 2 ** -8]))[0] == one + 2       # tie -> even (up)
    # just above a tie: an fp32 detour would round to the tie then to even (wrong)
    assert ref.round_bf16(np.array([1.0 + 2 ** -8 + 2 ** -40]))[0] == one + 1
    assert ref.round_bf16(np.array([-(1.0 + 2 ** -8 + 2 ** -40)]))[0] == (one + 1) | 0x8000


def test_bf16_to_f64_matches_torch_on_every_pattern():
    # every 16-bit pattern that is not a NaN, against torch's own bf16 -> fp32
    torch = pytest.importorskip("torch")
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    keep = ~np.isnan(t)
    assert keep.sum() == (1 << 16) - 2 * 127          # 127 NaN mantissas per sign
    np.testing.assert_array_equal(ref.bf16_to_f64(bits[keep]), t[keep].astype(np.float64))


# ------------------------------------------------------------------ SwiGLU activation
def test_silu_matches_scipy_expit():
    # silu(z) = z * sigmoid(z), against scipy's logistic function, up to |z| = 700
    sp = pytest.importorskip("scipy.special")
    z = np.concatenate([np.linspace(-700.0, 700.0, 20001), np.linspace(-8.0, 8.0, 4001),
                        [0.0, -0.0, 1e-300, -1e-300, 36.7, -36.7]])
    np.testing.assert_allclose(ref.silu(z), z * sp.expit(z), rtol=1e-14, atol=1e-300)


# ------------------------------------------------------------------ router
def test_router_logits_one_hot():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((16, 32)).astype(np.float32)
    b = rng.standard_normal(16).astype(np.float32)
    x = np.eye(32)[[3, 17]]
    l = ref.router_logits(x, W, b)
    np.testing.assert_array_equal(l, (W[:, [3, 17]].T.astype(np.float64) + b.astype(np.float64)))


def test_topk_matches_stable_argsort_and_ties():
    rng = np.random.default_rng(3)
    l = np.round(rng.standard_normal((64, 32)), 1)      # many exact ties
    for k in (1, 2, 8, 32):
        ids = ref.topk_ids(l, k)
        lib = np.argsort(-l, axis=1, kind="stable")[:, :k]
        np.testing.assert_array_equal(ids, lib)
    assert ref.topk_ids(np.array([[1.0, 3.0, 3.0, 0.0]]), 2).tolist() == [[1, 2]]


def test_gate_weights_sum_to_one_and_softmax_dense():
    sp = pytest.importorskip("scipy.special")
    rng = np.random.default_rng(4)
    l = rng.standard_normal((32, 16)) * 3
    for gating in (0, 1):
        ids = ref.topk_ids(l, 4)
        w = ref.gate_weights(l, ids, gating)
        np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-12)
        assert (w > 0).all()
        assert (np.diff(w, axis=1) <= 1e-15).all()      # largest logit first
    ids = ref.topk_ids(l, 16)                            # k = E: softmax MoE
    w = ref.gate_weights(l, ids, 0)
    dense = np.zeros_like(l)
    np.put_along_axis(dense, ids, w, axis=1)
    np.testing.assert_allclose(dense, sp.softmax(l, axis=1), rtol=1e-13, atol=0)
    w1 = ref.gate_weights(l, ids, 1)
    sig = sp.expit(np.take_along_axis(l, ids, 1))
    np.testing.assert_allclose(w1, sig / sig.sum(1, keepdims=True), rtol=1e-13)


def test_topk_gap():
    l = np.array([[5.0, 1.0, 4.0, 2.0], [0.0, 0.0, 0.0, 0.0]])
    np.testing.assert_array_equal(ref.topk_gap(l, 2), [2.0, 0.0])


# ------------------------------------------------------------------ permutation
def test_permutation_bijection_and_stable_order():
    rng = np.random.default_rng(6)
    for T, k, E in ((1, 8, 256), (64, 8, 256), (37, 2, 16)):
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
        counts, offsets, perm = ref.permutation(ids, E)
        assert counts.sum() == T * k and offsets[-1] == T * k
        np.testing.assert_array_equal(np.sort(perm), np.arange(T * k))
        np.testing.assert_array_equal(perm, np.argsort(ids.ravel(), kind="stable"))
        np.testing.assert_array_equal(counts, np.bincount(ids.ravel(), minlength=E))


# ------------------------------------------------------------------ whole layer
@pytest.mark.parametrize("variant", ["c0", "c0_shared_sigmoid"])
def test_sparse_equals_dense_bruteforce(variant):
    cfg = synth.TINY
    if variant == "c0_shared_sigmoid":
        cfg = cfg_with(cfg, n_shared=1, gating=1, top_k=3, tokens=6)
    layer = tiny_layer(cfg)
    x = synth.activations(cfg)
    sparse = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter)["out64"]
    dense = ref.dense_moe(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter)
    np.testing.assert_allclose(sparse, dense, rtol=1e-11, atol=1e-9 * np.abs(dense).max())


def test_zero_scale_experts_contribute_nothing():
    cfg = cfg_with(synth.TINY, n_shared=1)
    layer = tiny_layer(cfg, zero_routed=True)
    x = synth.activations(cfg)
    out = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 1, cfg.inter)["out64"]
    shared_only = ref.expert_ffn(ref.bf16_to_f64(x), *layer["experts"](cfg.n_experts), cfg.inter)
    np.testing.assert_allclose(out, shared_only, rtol=1e-12, atol=0)


def test_constant_weight_closed_form():
    # gate, up and down weights are the constants cg, cu, cd: with X = sum_h x_h,
    # g = cg*X and u = cu*X for every feature, h_i = silu(cg*X) * cu*X for all
    # i < I, y_o = cd * I * h, and the gate weights sum to 1.  Distinct constants
    # catch a swapped gate/up; the padded half of the down rows (I=128 < 256)
    # must not contribute.
    cg, cu, cd = 0.0625 * 2 * 5, 0.03125 * 3 * 7, 0.015625 * 1 * 11
    blocks = (make_block(0.0625, 0.75, [2] * 8, [0] * 8, [5] * 256),
              make_block(0.03125, 0.5, [3] * 8, [0] * 8, [7] * 256),
              make_block(0.015625, 0.25, [1] * 8, [0] * 8, [11] * 256))
    cfg = synth.TINY
    layer = tiny_layer(cfg, const_block=blocks)
    x = synth.activations(cfg)
    out = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 0, cfg.inter)["out64"]
    X = ref.bf16_to_f64(x).sum(1)
    expect = cd * cfg.inter * (cg * X / (1 + np.exp(-cg * X))) * (cu * X)
    np.testing.assert_allclose(out, np.repeat(expect[:, None], cfg.hidden, 1), rtol=1e-12)


def test_token_permutation_equivariance():
    cfg = cfg_with(synth.TINY, tokens=8, n_shared=1, gating=1)
    layer = tiny_layer(cfg)
    x = synth.activations(cfg)
    p = np.random.default_rng(0).permutation(cfg.tokens)
    a = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 1, cfg.inter)["out64"]
    b = ref.moe_forward(x[p], layer, cfg.top_k, cfg.gating, 1, cfg.inter)["out64"]
    np.testing.assert_allclose(b, a[p], rtol=1e-12, atol=1e-12 * np.abs(a).max())


def test_expert_relabelling_invariance():
    cfg = cfg_with(synth.TINY, tokens=6)
    layer = tiny_layer(cfg)
    x = synth.activations(cfg)
    E = cfg.n_experts
    sigma = np.random.default_rng(1).permutation(E)     # new label of old expert e is sigma[e]
    inv = np.argsort(sigma)
    relabelled = dict(router_w=layer["router_w"][inv], router_b=layer["router_b"][inv],
                      experts=lambda e: layer["experts"](int(inv[e]) if e < E else e))
    a = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 0, cfg.inter)
    b = ref.moe_forward(x, relabelled, cfg.top_k, cfg.gating, 0, cfg.inter)
    np.testing.assert_allclose(b["out64"], a["out64"], rtol=1e-12, atol=1e-12 * np.abs(a["out64"]).max())
    np.testing.assert_array_equal(np.sort(b["ids"], 1), np.sort(sigma[a["ids"]], 1))


def test_forced_routing_weights():
    cfg = cfg_with(synth.TINY, gating=1)
    layer = tiny_layer(cfg)
    x = synth.activations(cfg)
    forced = np.array([[0, 5], [1, 2], [15, 3], [7, 8]])
    r = ref.moe_forward(x, layer, 2, 1, 0, cfg.inter, forced_ids=forced)
    sig = 1 / (1 + np.exp(-np.take_along_axis(r["logits"], forced, 1)))
    np.testing.assert_allclose(r["w"], sig / sig.sum(1, keepdims=True), rtol=1e-14)
    np.testing.assert_array_equal(r["ids"], forced)


def test_token_subset_rows_equal_full_rows():
    # computing only some output rows gives those rows of the full run, in the
    # subset's order, with and without forced routing (the float rows up to
    # the summation order of the BLAS kernel, which depends on the row count)
    cfg = cfg_with(synth.TINY, tokens=9, n_shared=1, gating=1, top_k=3)
    layer = tiny_layer(cfg)
    x = synth.activations(cfg)
    subset = [7, 2, 5, 0]
    forced = np.random.default_rng(8).integers(0, cfg.n_experts, (cfg.tokens, cfg.top_k))
    for f in (None, forced):
        full = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 1, cfg.inter, forced_ids=f)
        part = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, 1, cfg.inter, forced_ids=f, token_subset=subset)
        np.testing.assert_array_equal(part["tokens"], subset)
        for key in ("out_bf16", "ids"):
            np.testing.assert_array_equal(part[key], full[key][subset], err_msg=key)
        for key in ("out64", "w", "logits", "gap"):
            np.testing.assert_allclose(part[key], full[key][subset], rtol=1e-12, atol=0, err_msg=key)


# ------------------------------------------------------------------ planted mistakes
def _pins_pass() -> bool:
    checks = [test_q4k_hand_block, test_q4k_closed_form_constant, test_q4k_weight_order,
              test_q4k_scale_pack_round_trip, test_topk_matches_stable_argsort_and_ties,
              test_gate_weights_sum_to_one_and_softmax_dense,
              lambda: test_sparse_equals_dense_bruteforce("c0_shared_sigmoid"),
              test_constant_weight_closed_form, test_permutation_bijection_and_stable_order,
              test_bf16_to_f64_matches_torch_on_every_pattern, test_silu_matches_scipy_expit,
              test_token_subset_rows_equal_full_rows, test_q8_0_closed_form, test_q5_k_fifth_bit_positions,
              test_q6_k_positions_and_offset, test_mxfp4_code_table_and_scale]
    checks += [lambda q=q: test_block_types_match_gguf_library(q) for q in (ref.Q5_K, ref.Q6_K, ref.Q8_0, ref.MXFP4)]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def _swap_nibbles(raw):
    raw = np.asarray(raw, np.uint8).copy()
    lead = raw.shape[:-1]
    b = raw.reshape(lead + (-1, 144))
    b[..., 16:] = ((b[..., 16:] >> 4) | (b[..., 16:] << 4)).astype(np.uint8)
    return raw


MUTANTS = {
    "nibble halves swapped": ("q4k_dequant", lambda orig: (lambda raw: orig(_swap_nibbles(raw)))),
    "min term dropped": ("q4k_scale_min", lambda orig: (lambda s: (orig(s)[0], 0 * orig(s)[1]))),
    "scale/min swapped": ("q4k_scale_min", lambda orig: (lambda s: orig(s)[::-1])),
    "ties to higher index": ("topk_ids", lambda orig: (lambda l, k: (l.shape[1] - 1 - orig(l[:, ::-1], k)))),
    "softmax over all logits": ("gate_weights", lambda orig: (
        lambda l, ids, g: orig(l, ids, g) if g else
        (np.exp(np.take_along_axis(l, ids, 1)) / np.exp(l).sum(1, keepdims=True)))),
    "silu on up instead of gate": ("expert_ffn", lambda orig: (
        lambda xr, g, u, d, inter, quants=(12, 12, 12): orig(xr, u, g, d, inter, quants))),
    "padding not masked": ("expert_ffn", lambda orig: (
        lambda xr, g, u, d, inter, quants=(12, 12, 12): _unmasked_ffn(xr, g, u, d))),
    "unstable permutation": ("permutation", lambda orig: (
        lambda ids, E: (lambda c, o, p: (c, o, p[::-1].copy()))(*orig(ids, E)))),
}


def _subset_forced_by_position(orig):
    # the bug: a subset run takes forced_ids row i for the subset's i-th token
    # instead of the row of that token
    def bad(x_bits, layer, k, gating, n_shared, inter, forced_ids=None, token_subset=None):
        if forced_ids is not None and token_subset is not None:
            f = np.asarray(forced_ids).copy()
            f[np.asarray(token_subset)] = np.asarray(forced_ids)[:len(token_subset)]
            forced_ids = f
        return orig(x_bits, layer, k, gating, n_shared, inter, forced_ids=forced_ids, token_subset=token_subset)
    return bad


def _q6k_offset16(orig):
    def bad(raw):
        b = np.asarray(raw, np.uint8).reshape(-1, 210)
        d = b[:, 208:210].copy().view(np.float16)[:, 0].astype(np.float64)
        sc = b[:, 192:208].view(np.int8).astype(np.float64)
        # the mistake: a zero point of 16 instead of 32
        w = orig(raw).reshape(-1, 256)
        scale = np.concatenate([np.concatenate([sc[:, 8 * h + 2 * p + np.arange(32) // 16] for p in range(4)], 1)
                                for h in range(2)], 1)
        return (w + d[:, None] * scale * 16.0).reshape(np.asarray(raw).shape[:-1] + (-1,))
    return bad


MUTANTS.update({
    "Q8_0 read as unsigned": ("q8_0_dequant", lambda orig: (lambda raw: (lambda b: (
        b[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)[..., None] *
        b[..., 2:34].astype(np.float64)).reshape(-1))(np.asarray(raw, np.uint8).reshape(-1, 34)))),
    "Q5_K fifth bits swapped": ("q5_k_dequant", lambda orig: (lambda raw: orig(_swap_q5_bits(raw)))),
    "Q6_K zero point 16": ("q6_k_dequant", _q6k_offset16),
    "MXFP4 bias 128": ("mxfp4_dequant", lambda orig: (lambda raw: 0.5 * orig(raw))),
    "bf16 shifted by 15": ("bf16_to_f64", lambda orig: (
        lambda bits: (np.asarray(bits, np.uint16).astype(np.uint32) << 15).view(np.float32).astype(np.float64))),
    "silu without the z factor": ("silu", lambda orig: (lambda z: 1.0 / (1.0 + np.exp(-z)))),
    "subset ignores its forced rows": ("moe_forward", _subset_forced_by_position),
})


def _swap_q5_bits(raw):
    # the mistake: fifth bit of the low nibble taken from bit 2c+1 and vice versa
    b = np.asarray(raw, np.uint8).reshape(-1, 176).copy()
    qh = b[:, 16:48].astype(np.int64)
    even, odd = qh & 0x55, (qh >> 1) & 0x55
    b[:, 16:48] = ((even << 1) | odd).astype(np.uint8)
    return b.reshape(np.asarray(raw).shape)


def _unmasked_ffn(xr, g, u, d):
    wg, wu, wd = ref.q4k_dequant(g), ref.q4k_dequant(u), ref.q4k_dequant(d)
    h = ref.silu(xr @ wg.T) * (xr @ wu.T)
    hp = np.zeros((h.shape[0], wd.shape[1]))
    hp[:, :h.shape[1]] = h
    hp[:, h.shape[1]:] = 1.0          # garbage in the pad: would leak through
    return hp @ wd.T


def test_pins_pass_on_the_real_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, monkeypatch):
    attr, make = MUTANTS[name]
    monkeypatch.setattr(ref, attr, make(getattr(ref, attr)))
    assert not _pins_pass(), f"planted mistake '{name}' went unnoticed"


# ------------------------------------------------------------------ other GGUF block types
def _sane_blocks(qtype, n, seed):
    """Random blocks of a GGUF type with finite scale fields."""
    rng = np.random.default_rng(seed)
    bs = ref.BLOCK[qtype][1]
    raw = rng.integers(0, 256, (n, bs), dtype=np.uint8)
    f16 = lambda v: np.asarray(v, np.float16).view(np.uint8).reshape(-1, 2)
    if qtype in (ref.Q5_K,):
        raw[:, 0:2] = f16(rng.uniform(-0.02, 0.02, n))
        raw[:, 2:4] = f16(rng.uniform(0, 0.01, n))
    elif qtype == ref.Q6_K:
        raw[:, 208:210] = f16(rng.uniform(-0.01, 0.01, n))
    elif qtype == ref.Q8_0:
        raw[:, 0:2] = f16(rng.uniform(-0.02, 0.02, n))
    elif qtype == ref.MXFP4:
        raw[:, 0] = rng.integers(110, 140, n)
    return raw.reshape(-1)


@pytest.mark.parametrize("qtype", [ref.Q5_K, ref.Q6_K, ref.Q8_0, ref.MXFP4])
def test_block_types_match_gguf_library(qtype):
    gguf = pytest.importorskip("gguf")
    from gguf.quants import dequantize
    raw = _sane_blocks(qtype, 64, qtype)
    ours = ref.dequant(raw, qtype)
    lib = dequantize(raw, gguf.GGMLQuantizationType(qtype)).astype(np.float64).reshape(ours.shape)
    np.testing.assert_allclose(ours, lib, rtol=1e-6, atol=1e-7 * np.abs(lib).max())


def test_q8_0_closed_form():
    blk = np.zeros(34, np.uint8)
    blk[0:2] = np.frombuffer(np.float16(0.25).tobytes(), np.uint8)
    blk[2:] = np.arange(-16, 16, dtype=np.int8).view(np.uint8)
    np.testing.assert_array_equal(ref.q8_0_dequant(blk), 0.25 * np.arange(-16, 16))


def test_q5_k_fifth_bit_positions():
    # all quants zero, one fifth bit set: exactly one weight becomes d*sc*16
    for pos in (0, 31, 32, 63, 64, 130, 255):
        blk = np.zeros(176, np.uint8)
        blk[0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
        blk[4:16] = pack_scales(np.ones((1, 8), np.int64), np.zeros((1, 8), np.int64))[0]
        c, rem = divmod(pos, 64)
        half, i = divmod(rem, 32)
        blk[16 + i] = 1 << (2 * c + half)
        w = ref.q5_k_dequant(blk)
        assert np.flatnonzero(w).tolist() == [pos] and w[pos] == 16.0


def test_q6_k_positions_and_offset():
    # ql = qh = 0 gives q - 32 = -32 everywhere; then one low nibble of 5 at
    # each byte lands on its documented position
    blk = np.zeros(210, np.uint8)
    blk[192:208] = np.arange(1, 17, dtype=np.int8).view(np.uint8)     # scale s = 1..16
    blk[208:210] = np.frombuffer(np.float16(0.5).tobytes(), np.uint8)
    base = ref.q6_k_dequant(blk)
    for h in (0, 1):
        for part in range(4):
            for i in (0, 17, 31):
                w = 128 * h + 32 * part + i
                g = i // 16 + 2 * part + 8 * h
                assert base[w] == 0.5 * (g + 1) * -32
    b2 = blk.copy()
    b2[64 + 40] = 0x05            # half 1, ql[40]: low nibble -> weight 128+32+8, high nibble -> 128+96+8
    w2 = ref.q6_k_dequant(b2)
    diff = np.flatnonzero(w2 != base).tolist()
    assert diff == [128 + 40]
    assert w2[168] == 0.5 * 11 * (5 - 32)   # scale index 8 + 0 + 2 = 10 -> s = 11


def test_mxfp4_code_table_and_scale():
    blk = np.zeros(17, np.uint8)
    blk[0] = 127 + 3                                       # 2^3
    blk[1:17] = (np.arange(16) | (np.arange(16)[::-1] << 4)).astype(np.uint8)
    w = ref.mxfp4_dequant(blk)
    e2m1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    np.testing.assert_array_equal(w[:16], 8.0 * np.array(e2m1))
    np.testing.assert_array_equal(w[16:], 8.0 * np.array(e2m1[::-1]))


@pytest.mark.parametrize("quants", [(13, 8, 14), (39, 39, 39), (14, 12, 8)])
def test_sparse_equals_dense_mixed_block_types(quants):
    cfg = cfg_with(synth.TINY, n_shared=1, gating=1, top_k=3, tokens=5, inter=300, quants=quants, seed=9)
    layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg),
                 experts=lambda e: synth.expert_tensors(cfg, 0, e), quants=quants)
    x = synth.activations(cfg)
    sparse = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter)["out64"]
    dense = ref.dense_moe(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter)
    np.testing.assert_allclose(sparse, dense, rtol=1e-11, atol=1e-9 * np.abs(dense).max())
    assert np.isfinite(sparse).all() and np.abs(sparse).max() > 0
