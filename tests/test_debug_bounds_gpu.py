"""The bounds-checking build (libmoe_debug.so, -DMOE_DEBUG_BOUNDS): every
index a kernel reads from memory -- expert ids, cache slots, row offsets,
permutation entries -- is checked before it addresses memory, and a bad one
is reported through moe_check.  Here the small layers run through that build
(in a child process: the variant is chosen when the library loads) on the
decode, batched and prefill paths and through a small streaming cache; no
check may fire, and the outputs still match the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import dataclasses, numpy as np, torch
from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import build, moe, synth
from routed_expert_ffn_forward_b200.layer import layer_from_config
from tests import parity_util as pu
assert moe.LIB_PATH.endswith("libmoe_debug.so")
build.build(debug_bounds=True)
cfgs = [synth.TINY, dataclasses.replace(synth.TINY, hidden=512, inter=300, n_experts=40, top_k=5, n_shared=2,
                                        gating=1, seed=13, router_std=1 / 512 ** 0.5)]
for cfg in cfgs:
    # resident, then streamed through a cache with room for every expert of
    # the layer (T = 17 may route to all of them)
    for stream_slots in (None, cfg.n_experts + cfg.n_shared + 2):
        moe.moe_set_cache_bytes(moe.SIZE_MAX if stream_slots is None
                                else stream_slots * moe.moe_expert_bytes(cfg.hidden, cfg.inter))
        L = layer_from_config(cfg)
        layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg),
                     experts=lambda e: synth.expert_tensors(cfg, 0, e))
        for T in (1, 3, 17):
            x = synth.activations(cfg, tokens=T)
            out = L.forward(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda())
            ids = L.routing(T)[0].cpu().numpy()
            torch.cuda.synchronize()
            moe.moe_check(L.handle)                # raises if a bounds check fired
            l64 = ref.router_logits(ref.bf16_to_f64(x), layer["router_w"], layer["router_b"])
            near = pu.check_ids(ids, l64, cfg.top_k)
            forced = np.where(near[:, None], ids, ref.topk_ids(l64, cfg.top_k))
            want = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
            pu.check_outputs(out.view(torch.int16).cpu().numpy().view(np.uint16), want["out_bf16"], cfg.name)
        L.destroy()
moe.moe_set_cache_bytes(moe.SIZE_MAX)
print("debug-bounds ok")
'''


def test_debug_bounds_build_runs_clean():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    env = dict(os.environ, MOE_LIB_VARIANT="debug", PYTHONPATH=ROOT)
    r = subprocess.run([sys.executable, "-c", CHILD], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug-bounds ok" in r.stdout
