"""Expert streaming through the device cache (GPU).

Streamed layers must give bit-identical outputs to resident layers (same
kernels, same arithmetic; only where the weights come from differs), and the
cache's hit/miss/eviction counts must match a host-side model of its LRU
policy step by step.  A small cache forces evictions every step.
"""
import dataclasses

import numpy as np
import pytest

from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import build, moe, synth
from tests import parity_util as pu
from tests.cache_model import CacheModel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    yield _t
    moe.moe_set_cache_bytes(moe.SIZE_MAX)


def to_dev(torch, bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_trace(torch, cfg, layers, trace, steps, prefetch, model=None):
    outs = []
    for s in range(steps):
        for l in range(cfg.n_layers):
            if prefetch:
                nl, ns = (l + 1, s) if l + 1 < cfg.n_layers else (0, s + 1)
                if ns < steps:
                    layers[nl].prefetch(trace[ns, nl])
                    if model:
                        model.prefetch(nl, trace[ns, nl].tolist())
            x = synth.activations(cfg, l, s, tokens=1)
            out = layers[l].forward_routed(to_dev(torch, x), trace[s, l][None])
            if model:
                model.forward(l, trace[s, l].tolist() + [cfg.n_experts + j for j in range(cfg.n_shared)])
            outs.append(out.view(torch.int16).cpu().numpy().view(np.uint16))
    torch.cuda.synchronize()
    return outs


SMALL = dataclasses.replace(synth.TINY, name="streaming small", n_shared=1, gating=1, n_layers=3,
                            steps=14, seed=21)


@pytest.mark.parametrize("policy", ["lru", "lfu"])
@pytest.mark.parametrize("prefetch", [False, True])
@pytest.mark.parametrize("slots", [4, 7, 40])
def test_streaming_matches_resident_and_cache_model(torch, prefetch, slots, policy):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = SMALL
    trace = synth.streaming_trace(cfg)
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    res = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
    want = run_trace(torch, cfg, res, trace, cfg.steps, prefetch=False)
    for L in res:
        L.destroy()
    eb = moe.moe_expert_bytes(cfg.hidden, cfg.inter)
    moe.moe_set_cache_bytes(slots * eb + 7)
    moe.moe_set_cache_policy(moe.MOE_CACHE_LFU if policy == "lfu" else moe.MOE_CACHE_LRU)
    try:
        layers = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
        moe.moe_reset_stats()
        model = CacheModel(slots, policy)
        got = run_trace(torch, cfg, layers, trace, cfg.steps, prefetch=prefetch, model=model)
        st = moe.moe_get_stats()
        for L in layers:
            L.destroy()
    finally:
        moe.moe_set_cache_bytes(moe.SIZE_MAX)
        moe.moe_set_cache_policy(moe.MOE_CACHE_LRU)
    for a, b in zip(got, want):
        np.testing.assert_array_equal(a, b)
    assert st["cache_slots"] == slots and st["slot_bytes"] == eb
    assert (st["cache_hits"], st["cache_misses"], st["prefetches"], st["evictions"]) == \
        (model.hits, model.misses, model.prefetches, model.evictions)
    assert st["h2d_bytes"] == (model.misses + model.prefetches) * eb
    touched = len({k for k in model.key if k is not None}) + model.evictions
    if touched > slots:
        assert model.evictions > 0


@pytest.mark.parametrize("T", [1, 2])
def test_streaming_c1_shapes_against_oracle(torch, T):
    """Full-size expert shapes (hidden 7168, inter 2048), 32 experts per layer,
    2 layers through a 20-slot cache (2 tokens need at most 17 experts);
    unrouted forwards (the routing is read back to the host before the
    experts are fetched, so one token takes the split decode kernels here)
    and a check of the last streamed output against the oracle."""
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = dataclasses.replace(synth.STREAMING, n_experts=32, n_layers=2, steps=6, seed=41)
    eb = moe.moe_expert_bytes(cfg.hidden, cfg.inter)
    moe.moe_set_cache_bytes(20 * eb)
    try:
        layers = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
        moe.moe_reset_stats()
        outs = []
        for s in range(3):
            for l in range(cfg.n_layers):
                x = synth.activations(cfg, l, s, tokens=T)
                o = layers[l].forward(to_dev(torch, x))
                ids, _ = layers[l].routing(T)
                outs.append((l, x, o.view(torch.int16).cpu().numpy().view(np.uint16), ids.cpu().numpy()))
        st = moe.moe_get_stats()
        for L in layers:
            L.destroy()
    finally:
        moe.moe_set_cache_bytes(moe.SIZE_MAX)
    assert st["cache_misses"] > 0 and st["evictions"] > 0
    l, x, o, ids = outs[-1]
    layer = dict(router_w=synth.router_weight(cfg, l), router_b=synth.router_bias(cfg, l),
                 experts=lambda e: synth.expert_tensors(cfg, l, e))
    l64 = ref.router_logits(ref.bf16_to_f64(x), layer["router_w"], layer["router_b"])
    near = pu.check_ids(ids, l64, cfg.top_k)
    forced = np.where(near[:, None], ids, ref.topk_ids(l64, cfg.top_k))
    r = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
    pu.check_outputs(o, r["out_bf16"], "streamed c1 shapes")


def test_streaming_full_shapes_sampled_against_oracle(torch):
    """The expert-streaming workload at its own shapes: 8 layers x (256 + 1)
    experts of hidden 7168 / inter 2048 in pinned host RAM (~51 GB), a
    12e9-byte cache (484 slots), the routing trace replayed through
    moe_forward_routed with next-layer prefetch for 40 steps (they touch ~560
    distinct experts, more than the slots, so slots are reused); four sampled
    (step, layer) outputs are compared with the oracle run on the same forced
    ids."""
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = synth.STREAMING
    steps = 40
    samples = [(3, 0), (17, 3), (29, 7), (39, 4)]
    trace = synth.streaming_trace(dataclasses.replace(cfg, steps=steps))
    eb = moe.moe_expert_bytes(cfg.hidden, cfg.inter)
    moe.moe_set_cache_bytes(cfg.cache_bytes)
    layers = []
    got = {}
    try:
        layers = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
        moe.moe_reset_stats()
        for s in range(steps):
            for l in range(cfg.n_layers):
                nl, ns = (l + 1, s) if l + 1 < cfg.n_layers else (0, s + 1)
                if ns < steps:
                    layers[nl].prefetch(trace[ns, nl])
                x = synth.activations(cfg, l, s, tokens=1)
                out = layers[l].forward_routed(to_dev(torch, x), trace[s, l][None])
                if (s, l) in samples:
                    got[(s, l)] = (x, out.view(torch.int16).cpu().numpy().view(np.uint16))
        torch.cuda.synchronize()
        for L in layers:
            moe.moe_check(L.handle)
        st = moe.moe_get_stats()
    finally:
        for L in layers:
            L.destroy()
            L.host = None
        moe.moe_set_cache_bytes(moe.SIZE_MAX)
        if hasattr(torch._C, "_host_emptyCache"):
            torch._C._host_emptyCache()     # give the 51 GB of pinned host memory back
    assert st["cache_slots"] == cfg.cache_bytes // eb == 484
    assert st["evictions"] > 0
    for (s, l), (x, out) in got.items():
        want = pu.oracle_rows(cfg, l, x, trace[s, l][None].astype(np.int64), [0], workers=1)
        pu.check_outputs(out, want, f"streamed step {s} layer {l}")


def test_cache_too_small_is_an_error(torch):
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = SMALL
    eb = moe.moe_expert_bytes(cfg.hidden, cfg.inter)
    moe.moe_set_cache_bytes(2 * eb)        # k + S = 3 experts per token
    try:
        L = layer_from_config(cfg, 0)
        x = synth.activations(cfg, 0, 0, tokens=1)
        with pytest.raises(moe.MoEError) as ei:
            L.forward_routed(to_dev(torch, x), np.array([[0, 1]], dtype=np.int32))
        assert ei.value.status == moe.MOE_ERR_CACHE_TOO_SMALL
        L.destroy()
        with pytest.raises(moe.MoEError) as ei:
            moe.moe_set_cache_bytes(eb - 1)
            layer_from_config(cfg, 0)
        assert ei.value.status == moe.MOE_ERR_CACHE_TOO_SMALL
    finally:
        moe.moe_set_cache_bytes(moe.SIZE_MAX)


def test_unpinned_host_memory_is_rejected(torch):
    cfg = SMALL
    h = moe.moe_layer_create(cfg.hidden, cfg.inter, cfg.n_experts, cfg.top_k, cfg.n_shared)
    buf = np.zeros(moe.moe_expert_bytes(cfg.hidden, cfg.inter), dtype=np.uint8)   # pageable
    p = [buf.ctypes.data] * (cfg.n_experts + cfg.n_shared)
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_set_experts(h, p, p, p)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_forward(h, 16, 16, 1, None)
    assert ei.value.status == moe.MOE_ERR_NOT_READY
    moe.moe_layer_destroy(h)


@pytest.mark.parametrize("T", [1, 2])
def test_streaming_block_types_against_oracle(torch, T):
    """Q6_K gate/up (210-byte blocks, copied into 224-byte device slots) and
    MXFP4 down (17-byte blocks grouped into 144 bytes) streamed through a small
    cache, routed on the GPU (read back before the experts are fetched)."""
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    cfg = dataclasses.replace(SMALL, quants=(14, 14, 39), inter=256, n_layers=2, seed=47)
    eb = moe.moe_expert_bytes(cfg.hidden, cfg.inter, 14)
    assert eb > 0
    moe.moe_set_cache_bytes(8 * max(eb, moe.moe_expert_bytes(cfg.hidden, cfg.inter, 39)))
    try:
        layers = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
        outs = []
        for s in range(4):
            for l in range(cfg.n_layers):
                x = synth.activations(cfg, l, s, tokens=T)
                o = layers[l].forward(to_dev(torch, x))
                ids, _ = layers[l].routing(T)
                outs.append((l, x, o.view(torch.int16).cpu().numpy().view(np.uint16), ids.cpu().numpy()))
        torch.cuda.synchronize()
        for L in layers:
            moe.moe_check(L.handle)
            L.destroy()
    finally:
        moe.moe_set_cache_bytes(moe.SIZE_MAX)
    for l, x, o, ids in outs[-2:]:
        layer = dict(router_w=synth.router_weight(cfg, l), router_b=synth.router_bias(cfg, l),
                     experts=lambda e, l=l: synth.expert_tensors(cfg, l, e), quants=cfg.quants)
        l64 = ref.router_logits(ref.bf16_to_f64(x), layer["router_w"], layer["router_b"])
        near = pu.check_ids(ids, l64, cfg.top_k)
        forced = np.where(near[:, None], ids, ref.topk_ids(l64, cfg.top_k))
        r = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
        pu.check_outputs(o, r["out_bf16"], f"streamed {cfg.quants}")
