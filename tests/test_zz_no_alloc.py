"""moe_route_noalloc: the router step for callers that cannot allocate device
memory (their device memory belongs to another allocator, or they cannot take
cudaMalloc's implicit synchronisation).

The GPU tests check it on two calls in a row against the CPU oracle's router
(logits, top-k, gating) and against the routing that moe_forward produces for
the same inputs; a second case runs without a bias, with 512 experts, on a
non-default stream, and follows a large call with a smaller one of another
expert count, so any read of the previous call's logits left in the shared
scratch array would change the result.  The argument checks run on the CPU:
they return before anything reaches the GPU.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes on its own in a
fresh process and after the other tests.
"""
import dataclasses

import numpy as np
import pytest

from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import build, moe, synth
from tests import parity_util as pu

CFG = dataclasses.replace(synth.BATCHED, name="no-alloc routing", hidden=1024, inter=256, n_experts=64,
                          top_k=6, tokens=40, seed=77, router_std=1 / 32)


def _torch_gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    return torch


def _check_against_oracle(x_bits, W, b, k, gating, ids, w):
    """Index rule and gate weights of the parity tests, against the oracle."""
    l64 = ref.router_logits(ref.bf16_to_f64(x_bits), W, b)
    pu.check_ids(ids, l64, k)
    w_or = ref.gate_weights(l64, ids.astype(np.int64), gating)
    np.testing.assert_allclose(w, w_or, rtol=1e-5, atol=1e-6)
    # ids ordered by decreasing logit
    sel = np.take_along_axis(l64, ids.astype(np.int64), 1)
    assert (np.diff(sel, axis=1) <= pu.GAP).all()


def _route(torch, x, W, b, T, H, E, k, gating, stream):
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), -1.0, dtype=torch.float32, device="cuda")
    moe.moe_route_noalloc(x.data_ptr(), W.data_ptr(), None if b is None else b.data_ptr(), T, H, E, k, gating,
                          ids.data_ptr(), w.data_ptr(), stream)
    return ids, w


@pytest.mark.gpu
def test_route_noalloc_matches_oracle_and_forward_twice():
    torch = _torch_gpu()
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    cfg = CFG
    L = layer_from_config(cfg)
    Wn, bn = synth.router_weight(cfg), synth.router_bias(cfg)
    W, b = torch.from_numpy(Wn).cuda(), torch.from_numpy(bn).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    try:
        for call in range(2):
            T = cfg.tokens - 7 * call          # second call: fewer tokens than the first
            x = synth.activations(cfg, 0, call, tokens=T)
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            L.forward(xd)
            ids_ref, w_ref = L.routing(T)
            ids, w = _route(torch, xd, W, b, T, cfg.hidden, cfg.n_experts, cfg.top_k, cfg.gating, stream)
            torch.cuda.synchronize()
            a, wa = ids.cpu().numpy(), w.cpu().numpy()
            _check_against_oracle(x, Wn, bn, cfg.top_k, cfg.gating, a, wa)
            # the existing entry point's routing: same sets outside the tie window
            r = ids_ref.cpu().numpy()
            l64 = ref.router_logits(ref.bf16_to_f64(x), Wn, bn)
            clear = ref.topk_gap(l64, cfg.top_k) >= pu.GAP
            np.testing.assert_array_equal(np.sort(a[clear], 1), np.sort(r[clear], 1))
            same = (a == r).all(1)
            np.testing.assert_allclose(wa[same], w_ref.cpu().numpy()[same], rtol=1e-5, atol=1e-6)
    finally:
        L.destroy()


@pytest.mark.gpu
def test_route_noalloc_no_bias_wide_experts_side_stream():
    torch = _torch_gpu()
    side = torch.cuda.Stream()
    # first call: 120 tokens x 512 experts fills 61440 of the 65536 scratch
    # floats; second call: 50 tokens x 300 experts, another router
    cases = [(dataclasses.replace(CFG, hidden=512, n_experts=512, top_k=8, gating=0, seed=78,
                                  router_std=1 / 512 ** 0.5, zipf_s=None), 120),
             (dataclasses.replace(CFG, hidden=768, n_experts=300, top_k=5, gating=1, seed=79,
                                  router_std=1 / 768 ** 0.5, zipf_s=None), 50)]
    for cfg, T in cases:
        Wn = synth.router_weight(cfg)
        x = synth.activations(cfg, 0, 0, tokens=T)
        with torch.cuda.stream(side):
            W = torch.from_numpy(Wn).to("cuda", non_blocking=False)
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to("cuda")
            ids, w = _route(torch, xd, W, None, T, cfg.hidden, cfg.n_experts, cfg.top_k, cfg.gating,
                            side.cuda_stream)
        side.synchronize()
        _check_against_oracle(x, Wn, None, cfg.top_k, cfg.gating, ids.cpu().numpy(), w.cpu().numpy())


def test_route_noalloc_rejects_oversize():
    pytest.importorskip("torch")
    build.build()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route_noalloc(16, 16, None, 257, 256, 256, 8, 1, 16, 16, None)   # 257*256 > 65536
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert "scratch" in moe.moe_last_error()


@pytest.mark.parametrize("offsets,what", [((4, 0, 0, 0, 0), "W"), ((0, 8, 0, 0, 0), "x"),
                                          ((0, 0, 2, 0, 0), "bias"), ((0, 0, 0, 1, 0), "ids"),
                                          ((0, 0, 0, 0, 2), "weights")])
def test_route_noalloc_rejects_misaligned_pointers(offsets, what):
    # rejected before anything is launched: the (fake) addresses are never touched
    pytest.importorskip("torch")
    build.build()
    base = 1 << 20
    dW, dx, db, di, dw = offsets
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route_noalloc(base + dx, base + dW, base + db, 4, 256, 16, 2, 1, base + di, base + dw, None)
    assert ei.value.status == moe.MOE_ERR_INVALID_ARG
    assert what in moe.moe_last_error()
