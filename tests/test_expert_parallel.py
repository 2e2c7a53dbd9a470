"""Expert parallelism: the experts are split across ranks (expert e on rank
e % world), each rank sums its own experts' contributions, the partials are
gathered in rank order and added in that order.

CPU part (no GPU): two gloo ranks run the exchange of ep.py with partials
the oracle computes for each rank's experts; the rank-order sum must equal
the oracle's whole layer (every pick counted on exactly one rank) and be the
same on both ranks.  GPU part: on one GPU, W ranks are emulated one after
another (each a layer told its rank), and the rank-order combine of their
partials is compared with the oracle and with the undivided layer."""
import dataclasses
import datetime
import os
import socket
import sys

import numpy as np
import pytest

from oracle import moe_ref as ref
from routed_expert_ffn_forward_b200 import synth
from tests import parity_util as pu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CFG = dataclasses.replace(synth.TINY, n_shared=2, gating=1, top_k=3, tokens=5, seed=51)


def oracle_partial(cfg, x, rank, world):
    """Sum, per token, of the weighted outputs of the experts rank owns
    (shared experts E.. included), from the oracle's pieces."""
    layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg),
                 experts=lambda e: synth.expert_tensors(cfg, 0, e))
    x64 = ref.bf16_to_f64(x)
    ids, w, _ = ref.route(x64, layer["router_w"], layer["router_b"], cfg.top_k, cfg.gating)
    out = np.zeros((x.shape[0], cfg.hidden))
    for t in range(x.shape[0]):
        for j in range(cfg.top_k):
            e = int(ids[t, j])
            if e % world == rank:
                out[t] += w[t, j] * ref.expert_ffn(x64[t:t + 1], *layer["experts"](e), cfg.inter)[0]
        for s in range(cfg.n_shared):
            if (cfg.n_experts + s) % world == rank:
                out[t] += ref.expert_ffn(x64[t:t + 1], *layer["experts"](cfg.n_experts + s), cfg.inter)[0]
    return out


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from routed_expert_ffn_forward_b200 import ep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        x = synth.activations(CFG)
        part = torch.from_numpy(oracle_partial(CFG, x, rank, world))
        gathered = ep.exchange(part).numpy()
        total = gathered[0].copy()
        for r in range(1, world):
            total += gathered[r]
        q.put((rank, gathered, total))
    finally:
        dist.destroy_process_group()


def test_exchange_two_gloo_ranks_partition_and_rank_order():
    import multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = synth.activations(CFG)
    want = ref.moe_forward(x, dict(router_w=synth.router_weight(CFG), router_b=synth.router_bias(CFG),
                                   experts=lambda e: synth.expert_tensors(CFG, 0, e)),
                           CFG.top_k, CFG.gating, CFG.n_shared, CFG.inter)["out64"]
    (_, g0, t0), (_, g1, t1) = res
    np.testing.assert_array_equal(g0, g1)                 # the same stack on both ranks
    np.testing.assert_array_equal(t0, t1)                 # the same rank-order sum
    np.testing.assert_allclose(g0[0], oracle_partial(CFG, x, 0, 2), rtol=0, atol=0)   # rank order
    np.testing.assert_allclose(t0, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


# ------------------------------------------------------------------ GPU: W ranks emulated on one GPU
EP_CFGS = {
    "small": CFG,
    "ragged": dataclasses.replace(synth.TINY, hidden=512, inter=300, n_experts=40, top_k=5, n_shared=2, gating=1,
                                  seed=52, router_std=1 / 512 ** 0.5),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", sorted(EP_CFGS))
@pytest.mark.parametrize("T", [1, 3, 17])
@pytest.mark.parametrize("world", [2, 3])
def test_emulated_ranks_match_oracle(name, T, world):
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from routed_expert_ffn_forward_b200 import build, moe
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    build.build()
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    cfg = EP_CFGS[name]
    L = layer_from_config(cfg)
    x = synth.activations(cfg, tokens=T)
    xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    try:
        whole = L.forward(xd).clone()
        ids = L.routing(T)[0].cpu().numpy()
        parts = torch.empty((world, T, cfg.hidden), dtype=torch.float32, device="cuda")
        for r in range(world):
            L.set_expert_parallel(r, world)
            L.forward_partial(xd, parts[r])
        out = torch.empty((T, cfg.hidden), dtype=torch.bfloat16, device="cuda")
        moe.moe_combine_partials(parts.data_ptr(), out.data_ptr(), T, cfg.hidden, world,
                                 torch.cuda.current_stream().cuda_stream)
        torch.cuda.synchronize()
        moe.moe_check(L.handle)
    finally:
        L.destroy()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg),
                 experts=lambda e: synth.expert_tensors(cfg, 0, e))
    l64 = ref.router_logits(ref.bf16_to_f64(x), layer["router_w"], layer["router_b"])
    near = pu.check_ids(ids, l64, cfg.top_k)
    forced = np.where(near[:, None], ids, ref.topk_ids(l64, cfg.top_k))
    want = ref.moe_forward(x, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced)
    pu.check_outputs(got, want["out_bf16"], f"EP world={world}")
    # the undivided layer: the same value up to the order of the fp32 sums
    pu.check_outputs(got, whole.view(torch.int16).cpu().numpy().view(np.uint16), "EP vs whole layer")
