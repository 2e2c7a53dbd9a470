"""moe_route_noalloc: the router step for callers that cannot allocate device
memory (their device memory belongs to another allocator, or they cannot take
cudaMalloc's implicit synchronisation), checked against the routing that
moe_forward produces for the same inputs, on two calls in a row.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It passes on its own in a
fresh process and after the other tests (the library's scratch array keeps
the previous call's logits, which must not leak into the next result).
"""
import dataclasses

import numpy as np
import pytest

from routed_expert_ffn_forward_b200 import build, moe, synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

CFG = dataclasses.replace(synth.BATCHED, name="no-alloc routing", hidden=1024, inter=256, n_experts=64,
                          top_k=6, tokens=40, seed=77, router_std=1 / 32)


def test_route_noalloc_matches_forward_routing_twice():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    cfg = CFG
    L = layer_from_config(cfg)
    W = torch.from_numpy(synth.router_weight(cfg)).cuda()
    b = torch.from_numpy(synth.router_bias(cfg)).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    try:
        for call in range(2):
            T = cfg.tokens - 7 * call          # second call: fewer tokens than the first
            x = synth.activations(cfg, 0, call, tokens=T)
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
            L.forward(xd)
            ids_ref, w_ref = L.routing(T)
            logits = L.logits(T)
            ids = torch.full((T, cfg.top_k), -1, dtype=torch.int32, device="cuda")
            w = torch.full((T, cfg.top_k), -1.0, dtype=torch.float32, device="cuda")
            moe.moe_route_noalloc(xd.data_ptr(), W.data_ptr(), b.data_ptr(), T, cfg.hidden, cfg.n_experts,
                                  cfg.top_k, cfg.gating, ids.data_ptr(), w.data_ptr(), stream)
            torch.cuda.synchronize()
            a, r = ids.cpu().numpy(), ids_ref.cpu().numpy()
            l64 = logits.cpu().numpy().astype(np.float64)
            gap = np.sort(l64, 1)[:, ::-1]
            gap = gap[:, cfg.top_k - 1] - gap[:, cfg.top_k]
            clear = gap >= pu.GAP                          # same index rule as the parity tests
            np.testing.assert_array_equal(np.sort(a[clear], 1), np.sort(r[clear], 1))
            same = (a == r).all(1)
            np.testing.assert_allclose(w.cpu().numpy()[same], w_ref.cpu().numpy()[same], rtol=1e-5, atol=1e-6)
            assert np.allclose(w.cpu().numpy().sum(1), 1.0, atol=1e-5)
    finally:
        L.destroy()


def test_route_noalloc_rejects_oversize():
    pytest.importorskip("torch")
    build.build()
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route_noalloc(16, 16, None, 257, 256, 256, 8, 1, 16, 16, None)   # 257*256 > 65536
    assert ei.value.status == moe.MOE_ERR_UNSUPPORTED
    assert "scratch" in moe.moe_last_error()
