"""Failure detection on the GPU without a GPU fault: the single-token kernel's
wait for the router's logits (where every CTA waits for all the others) is
told (a test hook) to look for the logits of the next launch, which no CTA
writes -- a flag that nothing sets.  Every CTA
gives up after a short limit, drains its copies in flight and exits; the
forward's stream and the context stay usable, moe_check reports the error
and resets the kernel's counters, and the next forward gives the same result
as before."""
import dataclasses

import numpy as np
import pytest

from routed_expert_ffn_forward_b200 import build, moe, synth

pytestmark = pytest.mark.gpu


def test_cross_cta_wait_runs_out_and_recovers():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    cfg = dataclasses.replace(synth.TINY, n_shared=1, gating=1, seed=31)
    L = layer_from_config(cfg)
    x = torch.from_numpy(synth.activations(cfg, tokens=1).view(np.int16)).view(torch.bfloat16).cuda()
    try:
        want = L.forward(x).clone()
        torch.cuda.synchronize()
        moe.moe_check(L.handle)
        moe.moe_set_test_hooks(20_000_000, 1)          # 20 ms, logits of a launch that never comes
        try:
            L.forward(x)
            torch.cuda.synchronize()                   # the kernel returns: nothing hangs
            with pytest.raises(moe.MoEError) as ei:
                moe.moe_check(L.handle)
            assert ei.value.status == moe.MOE_ERR_CUDA and "gave up" in str(ei.value)
        finally:
            moe.moe_set_test_hooks(0, 0)
        for _ in range(2):
            got = L.forward(x)
            torch.cuda.synchronize()
            moe.moe_check(L.handle)
            assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    finally:
        L.destroy()
