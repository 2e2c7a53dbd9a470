"""GPU parity: the CUDA path through the C ABI against the CPU oracle, on the
same seeded inputs.  Small shapes are compared element by element over every
token; the full-size configurations compare router ids over every token and
outputs over sampled tokens (the oracle computes those rows one by one)."""
import dataclasses

import numpy as np
import pytest

from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import build, moe, synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="session")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    moe.lib()
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    return _t


def oracle_layer(cfg, layer_index=0):
    return dict(router_w=synth.router_weight(cfg, layer_index), router_b=synth.router_bias(cfg, layer_index),
                experts=lambda e: synth.expert_tensors(cfg, layer_index, e))


def to_dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_bits(torch, t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_gpu(torch, cfg, T, layer_index=0, layer=None):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    L = layer or layer_from_config(cfg, layer_index)
    x = synth.activations(cfg, layer_index, tokens=T)
    out = L.forward(to_dev(torch, x))
    ids, w = L.routing(T)
    logits = L.logits(T)
    torch.cuda.synchronize()
    moe.moe_check(L.handle)   # no kernel gave up on a bounded wait
    res = dict(x=x, out=to_bits(torch, out), ids=ids.cpu().numpy(), w=w.cpu().numpy(),
               logits=logits.cpu().numpy())
    if layer is None:
        L.destroy()
    return res


def check_against_oracle(cfg, g, sample=None, layer_index=0, parallel=False):
    """Index rule on every token, outputs on `sample` tokens (all if None);
    with `parallel` the oracle rows are computed by several processes."""
    ol = oracle_layer(cfg, layer_index)
    x = g["x"]
    T = x.shape[0]
    l64 = ref.router_logits(ref.bf16_to_f64(x), ol["router_w"], ol["router_b"])
    np.testing.assert_allclose(g["logits"], l64, rtol=0, atol=1e-4 * max(1.0, np.abs(l64).max()))
    near = pu.check_ids(g["ids"], l64, cfg.top_k)
    toks = np.arange(T) if sample is None else np.asarray(sample)
    # weights of the GPU's picks, by the oracle's gating of its own logits
    w_or = ref.gate_weights(l64, g["ids"].astype(np.int64), cfg.gating)
    np.testing.assert_allclose(g["w"], w_or, rtol=1e-5, atol=1e-6)
    forced = np.where(near[:, None], g["ids"], ref.topk_ids(l64, cfg.top_k))
    if parallel:
        want = pu.oracle_rows(cfg, layer_index, x, forced, toks)
    else:
        want = ref.moe_forward(x, ol, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced,
                               token_subset=toks)["out_bf16"]
    return pu.check_outputs(g["out"][toks], want, cfg.name)


# ------------------------------------------------------------------ small shapes, every token
C0 = synth.TINY
SMALL = {
    "c0": C0,
    "c0_shared_sigmoid_bias": dataclasses.replace(C0, n_shared=1, gating=1, zipf_s=1.1, seed=11),
    "k_equals_E": dataclasses.replace(C0, top_k=16, seed=12),
    "ragged_inter": dataclasses.replace(C0, hidden=512, inter=300, n_experts=40, top_k=5, n_shared=2,
                                        gating=1, seed=13, router_std=1 / 512 ** 0.5),
    "k1_E1": dataclasses.replace(C0, n_experts=1, top_k=1, seed=14),
}


@pytest.mark.parametrize("name", sorted(SMALL))
@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 17, 64, 65, 200])
def test_small_every_token(torch, name, T):
    cfg = SMALL[name]
    g = run_gpu(torch, cfg, T)
    check_against_oracle(cfg, g)


@pytest.mark.parametrize("max_rows", [0, 1, 8, 32, 64])
def test_few_row_tile_thresholds(torch, max_rows):
    """The prefill path with the few-row kernel off (GEMM + decode kernels),
    taking only single-row experts, the experts up to 8 rows and the last
    partial tiles up to 8 rows, or everything up to 32 or 64 rows (the two
    builds of the kernel): every token
    matches the oracle each way (rows per expert 1..~60 here)."""
    cfg = SMALL["ragged_inter"]
    try:
        moe.moe_set_few_row_tiles(max_rows)
        g = run_gpu(torch, cfg, 200)
    finally:
        moe.moe_set_few_row_tiles(-1)
    check_against_oracle(cfg, g)


def test_zero_tokens(torch):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    L = layer_from_config(C0)
    x = torch.empty((0, C0.hidden), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, C0.hidden), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(L.handle, x.data_ptr(), out.data_ptr(), 0, None)
    L.destroy()


# ------------------------------------------------------------------ full-size configurations
def test_c1_decode_every_token(torch):
    cfg = synth.DECODE
    g = run_gpu(torch, cfg, cfg.tokens)
    check_against_oracle(cfg, g)


def test_c2_batched_decode_every_token(torch):
    cfg = synth.BATCHED
    g = run_gpu(torch, cfg, cfg.tokens)
    counts = np.bincount(g["ids"].ravel(), minlength=cfg.n_experts)
    assert (counts > 10).sum() >= 1 and (counts.max() <= cfg.tokens)
    check_against_oracle(cfg, g, parallel=True)


def prefill_sample(ids: np.ndarray, n_experts: int, tile: int = 256) -> np.ndarray:
    """Tokens whose rows reach every kind of work unit of the prefill path:
    the first and last row of every 256-row tile of the three experts with
    the most rows (full GEMM tiles and their last partial tile), one token of
    every expert with at most 64 rows (few-row tiles up to 32, small GEMM
    tiles above), and the last row of every expert whose last partial tile
    has at most 64 rows.  Rows of an expert are its (token, slot) pairs in
    token order."""
    T, k = ids.shape
    counts = np.bincount(ids.ravel(), minlength=n_experts)
    rows_of = {e: np.nonzero((ids == e).any(axis=1))[0] for e in range(n_experts) if counts[e]}
    pick = {0, T - 1}
    for e in np.argsort(-counts, kind="stable")[:3]:
        toks = rows_of[int(e)]
        for t0 in range(0, len(toks), tile):
            pick.add(int(toks[t0]))
            pick.add(int(toks[min(t0 + tile, len(toks)) - 1]))
    for e, toks in rows_of.items():
        if counts[e] <= 64:
            pick.add(int(toks[0]))
        elif 0 < counts[e] % tile <= 64:
            pick.add(int(toks[-1]))
    return np.array(sorted(pick))


def test_c3_prefill_sampled(torch):
    cfg = synth.PREFILL
    g = run_gpu(torch, cfg, cfg.tokens)
    sample = prefill_sample(g["ids"], cfg.n_experts)
    assert len(sample) >= 64
    check_against_oracle(cfg, g, sample=sample, parallel=True)


def test_single_token_deterministic(torch):
    """One token runs as one persistent kernel whose down units are claimed
    dynamically: the sums still run in a fixed order, so repeated forwards
    give identical bits; the routing read back matches the oracle."""
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = SMALL["ragged_inter"]
    L = layer_from_config(cfg)
    outs = []
    for rep in range(3):
        x = synth.activations(cfg, 0, rep % 2, tokens=1)
        outs.append(to_bits(torch, L.forward(to_dev(torch, x))))
    torch.cuda.synchronize()
    moe.moe_check(L.handle)
    np.testing.assert_array_equal(outs[0], outs[2])
    L.destroy()


def test_deterministic_and_host_path(torch):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = synth.BATCHED
    L = layer_from_config(cfg)
    x = synth.activations(cfg)
    xd = to_dev(torch, x)
    a = to_bits(torch, L.forward(xd))
    b = to_bits(torch, L.forward(xd))
    np.testing.assert_array_equal(a, b)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    moe.moe_forward_host(L.handle, xh.data_ptr(), oh.data_ptr(), cfg.tokens, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(oh.view(torch.int16).numpy().view(np.uint16), a)
    L.destroy()


@pytest.mark.parametrize("T", [1, 3, 4, 5])
def test_host_path_pinned_pageable_unaligned(torch, T):
    # decode sizes read and write pinned host buffers in place; pageable or
    # unaligned buffers, and T > 4, are copied: every route gives the device result
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = SMALL["c0_shared_sigmoid_bias"]
    L = layer_from_config(cfg)
    x = synth.activations(cfg, tokens=T)
    ref = to_bits(torch, L.forward(to_dev(torch, x)))
    n = T * cfg.hidden
    # pinned, aligned
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.full_like(xh, 7.0).pin_memory()
    moe.moe_forward_host(L.handle, xh.data_ptr(), oh.data_ptr(), T, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(oh.view(torch.int16).numpy().view(np.uint16).reshape(ref.shape), ref)
    # pageable
    xp = np.ascontiguousarray(x.view(np.uint16))
    op = np.zeros_like(xp)
    moe.moe_forward_host(L.handle, xp.ctypes.data, op.ctypes.data, T, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(op.reshape(ref.shape), ref)
    # pinned, 2 bytes off a 16-byte boundary
    xu = torch.zeros(n + 8, dtype=torch.bfloat16).pin_memory()
    ou = torch.zeros(n + 8, dtype=torch.bfloat16).pin_memory()
    xu[1:n + 1] = torch.from_numpy(x.view(np.int16).reshape(-1)).view(torch.bfloat16)
    moe.moe_forward_host(L.handle, xu.data_ptr() + 2, ou.data_ptr() + 2, T, None)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ou[1:n + 1].view(torch.int16).numpy().view(np.uint16).reshape(ref.shape), ref)
    moe.moe_check(L.handle)
    L.destroy()


def test_forced_routing(torch):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = SMALL["c0_shared_sigmoid_bias"]
    L = layer_from_config(cfg)
    x = synth.activations(cfg, tokens=5)
    forced = np.array([[0, 1], [15, 14], [3, 3], [7, 2], [9, 0]], dtype=np.int32)
    out = to_bits(torch, L.forward_routed(to_dev(torch, x), forced))
    ids, w = L.routing(5)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids.cpu().numpy(), forced)
    r = ref.moe_forward(x, oracle_layer(cfg), cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter,
                        forced_ids=forced)
    np.testing.assert_allclose(w.cpu().numpy(), r["w"], rtol=1e-5)
    pu.check_outputs(out, r["out_bf16"], "forced")
    with pytest.raises(moe.MoEError) as ei:
        L.forward_routed(to_dev(torch, x), np.full((5, 2), 16, dtype=np.int32))
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    L.destroy()


def test_large_weight_scales_are_exact(torch):
    """Q4_K blocks whose scales take weights far past the usual range: the
    prefill GEMMs dequantise to fp16 with a power-of-two scale chosen per
    weight row at moe_set_experts, so these rows are computed correctly too
    (no overflow, no flag); the decode kernels use the weights exactly."""
    from routed_expert_ffn_forward_b200.layer import MoELayer
    cfg = dataclasses.replace(C0, n_shared=1, gating=1, seed=15)

    def f16(v):
        return np.frombuffer(np.float16(v).tobytes(), dtype=np.uint8)

    def tensors(e):
        g, u, d = synth.expert_tensors(cfg, 0, e)
        g[0, 0:2] = f16(1.0)                              # |w| up to 945
        u[5, 0:2], u[5, 2:4] = f16(-2.0), f16(50.0)       # negative d, |w| up to 5040
        d[7, 2:4] = f16(1000.0)                           # |w| up to 63000: scale 2^-1
        d[9, 0:2] = f16(0.0)                              # d = 0, dmin only
        return g, u, d

    L = MoELayer(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k, cfg.n_shared)
    L.set_router(synth.router_weight(cfg), synth.router_bias(cfg), cfg.gating)

    def fill(e, views):
        for v, t in zip(views, tensors(e)):
            v[...] = t

    L.fill_experts(fill)
    L.register_experts()
    ol = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg), experts=tensors)
    for T in (1, 3, 256):       # decode (GEMV), decode (integer MMA), prefill (~32 rows per expert)
        x = synth.activations(cfg, tokens=T)
        out = to_bits(torch, L.forward(to_dev(torch, x)))
        ids, w = L.routing(T)
        logits = L.logits(T)
        torch.cuda.synchronize()
        moe.moe_check(L.handle)
        g = dict(x=x, out=out, ids=ids.cpu().numpy(), w=w.cpu().numpy(), logits=logits.cpu().numpy())
        l64 = ref.router_logits(ref.bf16_to_f64(x), ol["router_w"], ol["router_b"])
        near = pu.check_ids(g["ids"], l64, cfg.top_k)
        forced = np.where(near[:, None], g["ids"], ref.topk_ids(l64, cfg.top_k))
        r = ref.moe_forward(x, ol, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
        assert np.abs(r["out64"]).max() > 1e3          # the large rows dominate the output
        pu.check_outputs(out, r["out_bf16"], f"large scales, T={T}")
    L.destroy()


# ------------------------------------------------------------------ other GGUF block types
MIXED = {
    "q5k_q6k": dataclasses.replace(C0, n_shared=1, gating=1, quants=(13, 13, 14), seed=41),
    "q8_0_q8_0": dataclasses.replace(C0, hidden=512, inter=256, n_experts=24, top_k=3, n_shared=1, gating=1,
                                      quants=(8, 8, 8), seed=42, router_std=1 / 512 ** 0.5),
    "mxfp4_q4k": dataclasses.replace(C0, n_shared=2, gating=0, quants=(39, 39, 12), seed=43),
    "q4k_mxfp4": dataclasses.replace(C0, inter=256, quants=(12, 12, 39), seed=44),
    "q6k_q5k_ragged": dataclasses.replace(C0, hidden=512, inter=300, n_experts=40, top_k=5, n_shared=2, gating=1,
                                           quants=(14, 14, 13), seed=45, router_std=1 / 512 ** 0.5),
}


def mixed_oracle_layer(cfg, layer_index=0):
    d = oracle_layer(cfg, layer_index)
    d["quants"] = cfg.quants
    return d


@pytest.mark.parametrize("name", sorted(MIXED))
@pytest.mark.parametrize("T", [1, 3, 17])
def test_block_types_every_token(torch, name, T):
    """Layers whose weights are Q5_K, Q6_K, Q8_0 or MXFP4 (gate/up sharing a
    type, down another): every token runs the single-token kernel."""
    cfg = MIXED[name]
    g = run_gpu(torch, cfg, T)
    ol = mixed_oracle_layer(cfg)
    x = g["x"]
    l64 = ref.router_logits(ref.bf16_to_f64(x), ol["router_w"], ol["router_b"])
    np.testing.assert_allclose(g["logits"], l64, rtol=0, atol=1e-4 * max(1.0, np.abs(l64).max()))
    near = pu.check_ids(g["ids"], l64, cfg.top_k)
    np.testing.assert_allclose(g["w"], ref.gate_weights(l64, g["ids"].astype(np.int64), cfg.gating),
                               rtol=1e-5, atol=1e-6)
    forced = np.where(near[:, None], g["ids"], ref.topk_ids(l64, cfg.top_k))
    r = ref.moe_forward(x, ol, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
    pu.check_outputs(g["out"], r["out_bf16"], cfg.name + f" {cfg.quants}")


def test_block_types_c1_shapes(torch):
    """Full-size shapes (hidden 7168, inter 2048, 64 experts + 1 shared) with
    Q5_K gate/up and Q6_K down, one token, against the oracle."""
    cfg = dataclasses.replace(synth.DECODE, n_experts=64, quants=(13, 13, 14), seed=46)
    g = run_gpu(torch, cfg, 1)
    ol = mixed_oracle_layer(cfg)
    l64 = ref.router_logits(ref.bf16_to_f64(g["x"]), ol["router_w"], ol["router_b"])
    near = pu.check_ids(g["ids"], l64, cfg.top_k)
    forced = np.where(near[:, None], g["ids"], ref.topk_ids(l64, cfg.top_k))
    r = ref.moe_forward(g["x"], ol, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
    pu.check_outputs(g["out"], r["out_bf16"], "c1 shapes Q5_K/Q6_K")


def test_block_type_rejections(torch):
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_create_mixed(256, 128, 16, 2, 0, 12, 3)          # Q4_1 is not supported
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_layer_create_mixed(256, 300, 16, 2, 0, 12, 8)          # Q8_0 down needs inter % 256 == 0
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
