#!/usr/bin/env python
"""Benchmark of the routed mixture-of-experts FFN layer (libmoe.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config C]

Default workload (--config 1): MoE-layer decode, hidden 7168, inter 2048,
256 routed experts + 1 shared, top-8, sigmoid gating, T=1 token, all experts
resident in HBM.  One step = one moe_forward (router, permutation, gate/up +
SwiGLU, down, combine).  The L2 is flushed (a 256 MiB write) before every step
and only the forward is timed, with CUDA events on the forward's stream.
--config 2 (T=64), 3 (T=4096 prefill) and 4 (8-layer expert streaming with a
12e9-byte cache) run the other workloads.

Prints one JSON line (rank 0).  Under torchrun each rank runs an independent
replica on its own GPU (the layer has no cross-GPU exchange in this build), and
`value` is the tokens of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from routed_expert_ffn_forward_b200 import synth  # noqa: E402

CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------------------- helpers
class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    def __init__(self, device_index: int, directory: str):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join(directory, f"clocks_rank{device_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception as e:  # no nvidia-smi: report nothing rather than fail
            log("clock sampler unavailable:", e)
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            self.proc.wait(timeout=10)
            self.f.close()

    def summary(self) -> dict | None:
        if not self.proc:
            return None
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [q.strip() for q in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_traffic(key: str) -> float | None:
    """DRAM bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)
    of the kernel recorded under `key` ("config<N>:<kernel>") in
    profiles/traffic.json, if the kernel's source has not changed since the
    capture; None otherwise."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(key)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != d["sha256"]:
        return None
    return float(d["bytes_per_launch"])


def algorithmic_bytes(cfg, ids: np.ndarray, which: str) -> float:
    """Bytes a kernel must move at least once per launch for this routing.
    gate_up: gate+up weights of every expert the kernel runs, x rows, h writes.
    forward: every active expert's weights, the router weight, x and out.
    (The decode path, T <= 4, where every expert runs on one kernel.)"""
    T = ids.shape[0]
    active = len(np.unique(ids)) + cfg.n_shared
    nb_h, nb_i = cfg.hidden // 256, (cfg.inter + 255) // 256
    gate = cfg.inter * nb_h * 144
    down = cfg.hidden * nb_i * 144
    pairs = T * (cfg.top_k + cfg.n_shared)
    if which == "gate_up":
        return active * 2 * gate + T * cfg.hidden * 2 + pairs * cfg.inter * 2
    if which == "down":
        return active * down + pairs * cfg.inter * 2 + 2 * T * cfg.hidden * 2
    return active * (2 * gate + down) + cfg.n_experts * cfg.hidden * 4 + 2 * T * cfg.hidden * 2


def flops(cfg, T: int) -> float:
    return 2.0 * T * (cfg.top_k + cfg.n_shared) * 3 * cfg.hidden * cfg.inter


# ----------------------------------------------------------------------------- CPU oracle baseline
def _oracle_tokens(cfg, first: int, n_tokens: int, budget_s: float):
    """Whole tokens of the workload through the oracle (as it stands), one
    after another from token `first`, until the budget is used (at least
    one), BLAS limited to one thread.  Returns (tokens, seconds)."""
    from threadpoolctl import threadpool_limits

    from oracle import moe_ref as ref
    layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg),
                 experts=lambda e: synth.expert_tensors(cfg, 0, e))
    x = synth.activations(cfg, tokens=first + n_tokens)
    done, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=1):
        while done < n_tokens and (done == 0 or time.perf_counter() - t0 < budget_s):
            t = first + done
            ref.moe_forward(x[t:t + 1], layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter)
            done += 1
    return done, time.perf_counter() - t0


def _oracle_worker(job):
    cfg_index, first, n_tokens, budget_s = job
    return _oracle_tokens(synth.WORKLOADS[cfg_index], first, n_tokens, budget_s)


def oracle_sample_rate(cfg_index: int, n_tokens: int, budget_s: float) -> dict:
    """The oracle on one host core: whole tokens, one after another."""
    cfg = synth.WORKLOADS[cfg_index]
    done, dt = _oracle_tokens(cfg, 0, n_tokens, budget_s)
    return {"value": done / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{done} token(s) of the workload's layer through the fp64 numpy oracle "
                      f"(full routing + {cfg.top_k}+{cfg.n_shared} experts each), BLAS limited to 1 thread",
            "seconds": dt}


def oracle_all_cores(cfg_index: int, budget_s: float, max_workers: int = 16) -> dict:
    """The oracle on the host's cores: one spawned process per core (at most
    `max_workers`: each holds ~1 GB of fp64 weights), each running whole
    tokens of its own with BLAS limited to one thread, for about `budget_s`.
    value = all workers' tokens / the longest worker's time."""
    import multiprocessing as mp
    cfg = synth.WORKLOADS[cfg_index]
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    workers = max(1, min(cores, max_workers))
    jobs = [(cfg_index, 64 * w, 64, budget_s) for w in range(workers)]
    t0 = time.perf_counter()
    with mp.get_context("spawn").Pool(workers) as pool:
        res = pool.map(_oracle_worker, jobs)
    wall = time.perf_counter() - t0
    tokens = sum(r[0] for r in res)
    secs = max(r[1] for r in res)
    return {"value": tokens / secs, "unit": "tokens/s", "cores": workers, "kind": "oracle",
            "sample": f"{tokens} tokens of the workload's layer through the fp64 numpy oracle on {workers} "
                      f"processes (one per core, {cores} cores available, BLAS 1 thread each), "
                      f"~{budget_s:.0f} s each",
            "seconds": secs, "wall_s": wall}


_EXPERT_CACHE: dict = {}


def oracle_unit(cfg, step: int, rows_frac: float, ref, x64, l64):
    """One reference step: the oracle's expert FFN for token 0 restricted to one
    256-feature block of one of its experts (gate/up rows of that block, the
    down column block; rows_frac < 1 also subsamples rows).  Returns the
    fraction of one token's expert work it covers."""
    k, S = cfg.top_k, cfg.n_shared
    ids = ref.topk_ids(l64[:1], k)[0].tolist() + [cfg.n_experts + s for s in range(S)]
    e = ids[step % len(ids)]
    nb_i = (cfg.inter + 255) // 256
    b = (step // len(ids)) % nb_i
    if e not in _EXPERT_CACHE:
        _EXPERT_CACHE[e] = synth.expert_tensors(cfg, 0, e)
    g, u, d = _EXPERT_CACHE[e]
    r = max(1, int(round(min(256, cfg.inter - 256 * b) * rows_frac)))
    rows = slice(256 * b, 256 * b + r)
    wg, wu = ref.q4k_dequant(g[rows]), ref.q4k_dequant(u[rows])
    h = ref.silu(wg @ x64[0]) * (wu @ x64[0])
    ro = max(1, int(round(cfg.hidden * rows_frac)))
    wd = ref.q4k_dequant(d[:ro, 144 * b:144 * (b + 1)])[:, :r]
    _ = wd @ h
    total_blocks = len(ids) * (2 * cfg.inter * (cfg.hidden // 256) + cfg.hidden * nb_i)
    return (2 * r * (cfg.hidden // 256) + ro) / total_blocks


def run_reference(args, cfg) -> dict:
    """--impl reference: the oracle on the host cores, same metric and config."""
    from threadpoolctl import threadpool_limits

    from oracle import moe_ref as ref
    layer = dict(router_w=synth.router_weight(cfg), router_b=synth.router_bias(cfg))
    x = synth.activations(cfg, tokens=1)
    x64 = ref.bf16_to_f64(x)
    budget = 150.0
    rows_frac = min(1.0, budget / max(1, args.steps + args.warmup) / 0.09)
    fracs, times = [], []
    with threadpool_limits(limits=1):
        for step in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            l64 = ref.router_logits(x64, layer["router_w"], layer["router_b"])
            f = oracle_unit(cfg, step, rows_frac, ref, x64, l64)
            dt = time.perf_counter() - t0
            if step >= args.warmup:
                fracs.append(f)
                times.append(dt)
    tokens = float(np.sum(fracs))
    secs = float(np.sum(times))
    value = tokens / secs
    sample = (f"per step: router logits for one token plus one 256-feature block of one of its "
              f"{cfg.top_k + cfg.n_shared} experts (gate/up rows x{rows_frac:.3f}, down rows x{rows_frac:.3f}); "
              f"value = fraction of a token's expert work per second")
    return {"metric": "moe_layer_decode_tokens_per_s", "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, args),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_json(cfg, args) -> dict:
    return {"workload": cfg.name, "hidden": cfg.hidden, "inter": cfg.inter, "experts": cfg.n_experts,
            "top_k": cfg.top_k, "shared": cfg.n_shared, "tokens": cfg.tokens, "quant": "Q4_K",
            "gating": "softmax-topk" if cfg.gating == 0 else "sigmoid-renorm",
            "layers": cfg.n_layers, "cache_bytes": cfg.cache_bytes,
            "l2": "flushed before every step (256 MiB write)" if args.config != 4 else
                  "not flushed; working set 51 GB streamed through a 12e9 B cache",
            "parallelism": f"replicas x{args.gpus}"}


# ----------------------------------------------------------------------------- GPU arm
DTYPE_DECODE = "q4_k x fx16 -> i32"      # exact Q4_K weights, 16-bit fixed-point activations, int32 sums
DTYPE_PREFILL = "q4_k->f16 x f16 -> f32"  # Q4_K dequantised to fp16 (power-of-two scaled), fp32 accumulate


def measure_resident(args, cfg, rank, world, local_rank, peaks, steps, warmup, e2e=True) -> dict:
    """Time `steps` forwards of one resident layer of `cfg` (after `warmup`),
    L2 flushed before each, CUDA events on the forward's stream; then the same
    steps again with per-kernel profiling events, and optionally the
    end-to-end host-buffer path."""
    import torch

    from routed_expert_ffn_forward_b200 import moe
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    t0 = time.time()
    L = layer_from_config(cfg)
    log(f"[rank {rank}] layer '{cfg.name}' ready in {time.time() - t0:.1f}s")
    T = cfg.tokens
    n_pool = 16 if T > 1 else 64
    xs = [synth.activations(cfg, 0, i, tokens=T) for i in range(n_pool)]
    x_dev = torch.from_numpy(np.stack(xs).view(np.int16)).view(torch.bfloat16).to(dev)
    out = torch.empty((T, cfg.hidden), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    # routing of every pool entry (for the algorithmic byte counts)
    ids_pool = []
    for i in range(n_pool):
        L.forward(x_dev[i], out)
        ids_pool.append(L.routing(T)[0].cpu().numpy())
    torch.cuda.synchronize()

    def step(i, prof_events):
        flush.zero_()
        s, e = prof_events
        s.record(stream)
        L.forward(x_dev[i % n_pool], out, stream.cuda_stream)
        e.record(stream)

    for i in range(warmup):
        step(i, (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    st0 = moe.moe_get_stats()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank, args.clocks_dir) as clk:
        for i in range(steps):
            step(i, evs[i])
        torch.cuda.synchronize()
    barrier(world)
    st1 = moe.moe_get_stats()
    step_ms = [s.elapsed_time(e) for s, e in evs]
    total_ms = max_over_ranks(float(np.sum(step_ms)), world, dev)
    launches = st1["launches"] - st0["launches"]
    moe.moe_check(L.handle)
    # Per-kernel device times: the same steps again with the library recording
    # CUDA events around each kernel on the forward's stream.  (Events between
    # the chained kernels stop them from overlapping, so this pass is not the
    # one whose time is reported as `value`.)
    moe.moe_reset_profile()
    moe.moe_set_profiling(True)
    for i in range(steps):
        step(i, (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
    torch.cuda.synchronize()
    moe.moe_set_profiling(False)
    prof = moe.moe_get_profile()

    e2e_res = None
    if e2e:
        # the same forward through moe_forward_host, host buffers in and out
        xh = torch.from_numpy(np.stack(xs).view(np.int16)).view(torch.bfloat16).pin_memory()
        oh = torch.empty((T, cfg.hidden), dtype=torch.bfloat16).pin_memory()
        e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(steps)]
        for i in range(min(warmup, 3)):
            moe.moe_forward_host(L.handle, xh[i].data_ptr(), oh.data_ptr(), T, stream.cuda_stream)
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            s, e = e2e_evs[i]
            s.record(stream)
            moe.moe_forward_host(L.handle, xh[i % n_pool].data_ptr(), oh.data_ptr(), T, stream.cuda_stream)
            e.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(float(np.sum([s.elapsed_time(e) for s, e in e2e_evs])), world, dev)
        e2e_res = {"value": T * steps * world / (e2e_ms / 1e3), "unit": "tokens/s",
                   "h2d_bytes_per_step": T * cfg.hidden * 2, "d2h_bytes_per_step": T * cfg.hidden * 2,
                   "api": "moe_forward_host (pinned host x and out)"}
    L.destroy()
    L.host = None
    del flush, x_dev

    ids_cycle = [ids_pool[i % n_pool] for i in range(steps)]
    fwd_ms = total_ms / steps
    kern = "gate_up"
    avg_ms = prof["ms"][kern] / max(1, prof["launches"][kern])
    gemm_dominant = prof["ms"]["gate_up"] >= prof["ms"].get("few_gate_up", 0.0)
    if T > 4 and not gemm_dominant:
        # the few-row kernel carries the step: bound by HBM
        kern = "few_gate_up"
        avg_ms = prof["ms"][kern] / max(1, prof["launches"][kern])
        ab = float(np.mean([few_gate_up_bytes(cfg, ids) for ids in ids_cycle]))
        achieved = ab / (avg_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": kern, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": kernel_traffic(f"config{cfg_index(cfg)}:{kern}"),
                "algorithmic_bytes": ab, "peak_source": peaks["source"]}
    elif T > 4:
        # the gate/up GEMM runs the experts with more than 4 rows (plus the shared one)
        fl = float(np.mean([gate_up_gemm_flops(cfg, ids) for ids in ids_cycle]))
        achieved = fl / (avg_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops_sustained"] or peaks["bf16_tflops"]
        roof = {"bound": "tensor", "kernel": kern, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_burst_peak": achieved / peaks["bf16_tflops"],
                "flops_per_launch": fl, "traffic": kernel_traffic(f"config{cfg_index(cfg)}:{kern}"),
                "peak_source": peaks["source"] + " (sustained bf16; fp16 has the same nominal rate)"}
    else:
        if prof["launches"].get("fused"):
            # one token: the whole forward is one kernel, which moves every byte
            kern = "fused"
            avg_ms = prof["ms"][kern] / max(1, prof["launches"][kern])
        ab = float(np.mean([algorithmic_bytes(cfg, ids, "forward" if kern == "fused" else kern)
                            for ids in ids_cycle]))
        achieved = ab / (avg_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "kernel": kern, "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": kernel_traffic(f"config{cfg_index(cfg)}:{kern}"),
                "algorithmic_bytes": ab, "peak_source": peaks["source"]}
    fwd_bytes = float(np.mean([algorithmic_bytes(cfg, ids, "forward") for ids in ids_cycle]))
    steps_k = [q for q in moe.KERNELS if q != "forward"]
    kernels = {k: {"avg_us": 1e3 * prof["ms"][k] / max(1, prof["launches"][k]),
                   "share": prof["ms"][k] / max(1e-12, sum(prof["ms"][q] for q in steps_k))}
               for k in steps_k if prof["launches"][k]}
    return {"value": T * steps * world / (total_ms / 1e3), "ms_per_step": fwd_ms, "roofline": roof,
            "forward_hbm": {"algorithmic_bytes": fwd_bytes, "achieved_gbs": fwd_bytes / (fwd_ms / 1e3) / 1e9,
                            "frac": fwd_bytes / (fwd_ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
            "tflops": flops(cfg, T) / (fwd_ms / 1e3) / 1e12, "kernels": kernels, "e2e": e2e_res,
            "gpu_launches": launches, "clocks": clk.summary(),
            "dtype": DTYPE_DECODE if T <= 4 else DTYPE_PREFILL}


def few_rows_default(T: int) -> int:
    """The library's default moe_set_few_row_tiles for a batch of T tokens."""
    return 64 if T <= 256 else 32


def tile_split(cfg, ids: np.ndarray, few_rows: int | None = None):
    """How the prefill path splits this routing (as the library's tile
    builder does): (rows on the tensor-memory GEMM, rows on few-row tiles,
    number of few-row tiles).  An expert with at most few_rows rows is one
    few-row tile; a larger one goes to the GEMM in 256-row tiles, except a
    last partial tile of at most few_rows rows, which becomes a few-row tile."""
    T = ids.shape[0]
    counts = np.bincount(ids.ravel(), minlength=cfg.n_experts)
    few = few_rows_default(T) if few_rows is None else few_rows
    return split_rows([int(c) for c in counts if c > 0] + [T] * cfg.n_shared, few)


def split_rows(rows, few_rows: int = 32):
    """tile_split on a list of rows per active expert."""
    gemm = few = n_few = 0
    for c in rows:
        if c <= few_rows:
            few, n_few = few + c, n_few + 1
            continue
        last = c - (c - 1) // 256 * 256
        if last <= few_rows:
            gemm, few, n_few = gemm + c - last, few + last, n_few + 1
        else:
            gemm += c
    return gemm, few, n_few


def gate_up_gemm_flops(cfg, ids: np.ndarray) -> float:
    """FLOPs of the prefill gate/up GEMM for this routing: 2 * rows * 2I * H
    over the rows in its tiles (tile_split)."""
    return 2.0 * tile_split(cfg, ids)[0] * 2 * cfg.inter * cfg.hidden


def few_gate_up_bytes(cfg, ids: np.ndarray) -> float:
    """Bytes the few-row gate/up kernel moves at least once: the gate and up
    weights of every few-row tile, its x rows (fp16) and its h rows (fp32)."""
    _, few, n_few = tile_split(cfg, ids)
    gate = cfg.inter * (cfg.hidden // 256) * 144
    i_pad = (cfg.inter + 255) // 256 * 256
    return n_few * 2 * gate + few * cfg.hidden * 2 + few * i_pad * 4


def cfg_index(cfg) -> int:
    for k, v in synth.WORKLOADS.items():
        if v.name == cfg.name:
            return k
    return -1


def run_ours(args, cfg, rank: int, world: int, local_rank: int) -> dict | None:
    import torch

    from routed_expert_ffn_forward_b200 import build

    build.build()
    torch.cuda.set_device(local_rank)
    peaks = measured_peaks()
    if args.config == 4:
        return run_streaming(args, cfg, rank, world, local_rank, peaks)
    m = measure_resident(args, cfg, rank, world, local_rank, peaks, args.steps, args.warmup)
    T = cfg.tokens
    metric = "moe_layer_prefill_tokens_per_s" if args.config == 3 else "moe_layer_decode_tokens_per_s"
    res = {"metric": metric, "value": m["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": m["dtype"], "data": "synthetic", "config": config_json(cfg, args),
           "roofline": m["roofline"], "forward_hbm": m["forward_hbm"],
           "prefill_tflops": m["tflops"] if T > 4 else None, "kernels": m["kernels"], "e2e": m["e2e"],
           "gpu_launches": m["gpu_launches"], "clocks": m["clocks"]}
    if args.config == 1 and not args.no_extra and not args.small:
        # the batched-decode and prefill workloads of the same layer shape, one
        # resident layer at a time, same steps and warm-up
        for key, idx in (("batched", 2), ("prefill", 3)):
            c = synth.WORKLOADS[idx]
            x = measure_resident(args, c, rank, world, local_rank, peaks, args.steps, args.warmup, e2e=False)
            res[key] = {"workload": c.name, "tokens": c.tokens, "tokens_per_s": x["value"],
                        "ms_per_step": x["ms_per_step"], "tflops": x["tflops"], "forward_hbm": x["forward_hbm"],
                        "roofline": x["roofline"], "kernels": x["kernels"], "gpu_launches": x["gpu_launches"],
                        "clocks": x["clocks"], "dtype": x["dtype"]}
        res["prefill_tflops"] = res["prefill"]["tflops"]
        res["gpu_launches"] += res["batched"]["gpu_launches"] + res["prefill"]["gpu_launches"]
    return res


STREAM_MODES = ("lru+demand", "lfu+demand", "lru+trace", "lfu+trace")
EXTRA_STREAM_MODES = ("lfu+lookahead",)   # run only when named in --stream-modes


def run_streaming(args, cfg, rank, world, local_rank, peaks) -> dict:
    """Config 4: 8 stacked layers streamed through a 12e9-byte cache, one
    token per layer with the trace's routing.  Each mode empties the cache,
    runs the warm-up steps, then times the steps:
      <policy>+demand     misses are fetched when a forward needs them
      <policy>+trace      while layer l runs, layer l+1's experts are read from
                          the trace and prefetched: an oracle predictor, an
                          upper bound
      lfu+lookahead       (only when named) layer l+1's router
                          (moe_route_noalloc, on a high-priority side stream)
                          is applied to layer l's input, and while layer l
                          runs the experts it picks are prefetched: a
                          predictor that reads nothing of the future
    with policy lru or lfu (moe_set_cache_policy).  `value` is the fastest
    mode that does not read the trace.  (The workload's routing is a trace
    with its own temporal correlation, not the output of the layers'
    routers, and each (step, layer) input is a fresh draw, so the lookahead
    predictor sees nothing that the trace follows: it guesses at random here,
    and the cache's recency and frequency are the causal predictors this
    trace rewards.)"""
    import torch

    from routed_expert_ffn_forward_b200 import moe
    from routed_expert_ffn_forward_b200.layer import layer_from_config
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    h2d_peak = h2d_probe(dev)
    moe.moe_set_cache_bytes(cfg.cache_bytes)
    t0 = time.time()
    layers = [layer_from_config(cfg, l) for l in range(cfg.n_layers)]
    log(f"[rank {rank}] {cfg.n_layers} layers ready in {time.time() - t0:.1f}s")
    trace = synth.streaming_trace(cfg)
    warmup = max(args.warmup, 60)            # the cache and its counts settle
    n_steps = warmup + args.steps
    assert n_steps <= cfg.steps, f"trace has {cfg.steps} steps"
    xs = np.stack([synth.activations(cfg, l, s, tokens=1) for s in range(n_steps) for l in range(cfg.n_layers)])
    x_dev = torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16).to(dev).view(n_steps, cfg.n_layers, 1, -1)
    out = torch.empty((1, cfg.hidden), dtype=torch.bfloat16, device=dev)
    modes = args.stream_modes.split(",") if args.stream_modes else list(STREAM_MODES)
    for m in modes:
        if m not in STREAM_MODES + EXTRA_STREAM_MODES:
            raise SystemExit(f"unknown streaming mode {m!r}; choose from "
                             f"{','.join(STREAM_MODES + EXTRA_STREAM_MODES)}")
    if "lfu+lookahead" in modes:
        Ws = [torch.from_numpy(synth.router_weight(cfg, l)).to(dev) for l in range(cfg.n_layers)]
        bs = [torch.from_numpy(synth.router_bias(cfg, l)).to(dev) for l in range(cfg.n_layers)]
        p_ids = torch.empty((1, cfg.top_k), dtype=torch.int32, device=dev)
        p_w = torch.empty((1, cfg.top_k), dtype=torch.float32, device=dev)
        p_host = torch.empty((1, cfg.top_k), dtype=torch.int32).pin_memory()
        side = torch.cuda.Stream(dev, priority=-1)   # the predictor's router, beside the layer's forward
        p_done = torch.cuda.Event()

    def run_step(s, how):
        for l in range(cfg.n_layers):
            nl, ns = (l + 1, s) if l + 1 < cfg.n_layers else (0, s + 1)
            if how == "lookahead":
                # route layer l's input with layer l+1's router on the side
                # stream, queue layer l, then prefetch while layer l runs
                moe.moe_route_noalloc(x_dev[s, l].data_ptr(), Ws[nl].data_ptr(), bs[nl].data_ptr(), 1, cfg.hidden,
                                      cfg.n_experts, cfg.top_k, cfg.gating, p_ids.data_ptr(), p_w.data_ptr(),
                                      side.cuda_stream)
                with torch.cuda.stream(side):
                    p_host.copy_(p_ids, non_blocking=True)
                    p_done.record(side)
            layers[l].forward_routed(x_dev[s, l], trace[s, l][None], out, stream.cuda_stream)
            if how == "trace" and ns < n_steps:
                layers[nl].prefetch(trace[ns, nl])
            elif how == "lookahead":
                p_done.synchronize()
                layers[nl].prefetch(p_host.numpy()[0])

    res = {}
    clocks = None
    for mode in modes:
        policy, how = mode.split("+")
        moe.moe_set_cache_bytes(cfg.cache_bytes)          # empty cache
        moe.moe_set_cache_policy(moe.MOE_CACHE_LFU if policy == "lfu" else moe.MOE_CACHE_LRU)
        for s in range(warmup):
            run_step(s, how)
        torch.cuda.synchronize()
        moe.moe_reset_stats()
        barrier(world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local_rank, args.clocks_dir) as clk:
            ev0.record(stream)
            for s in range(warmup, n_steps):
                run_step(s, how)
            ev1.record(stream)
            torch.cuda.synchronize()
        st = moe.moe_get_stats()
        ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
        secs = ms / 1e3
        lookups = st["cache_hits"] + st["cache_misses"]
        res[mode] = {"tokens_per_s": args.steps * world / secs, "ms_per_step": ms / args.steps,
                     "hit_rate": st["cache_hits"] / max(1, lookups), "misses_per_step": st["cache_misses"] / args.steps,
                     "prefetches_per_step": st["prefetches"] / args.steps,
                     "h2d_gb_per_step": st["h2d_bytes"] / args.steps / 1e9, "h2d_gbs": st["h2d_bytes"] / secs / 1e9,
                     "h2d_frac": st["h2d_bytes"] / secs / 1e9 / h2d_peak, "gpu_launches": st["launches"],
                     "clocks": clk.summary()}
        clocks = clocks or res[mode]["clocks"]
        log(f"[rank {rank}] {mode}: {res[mode]['tokens_per_s']:.1f} tok/s, hit rate {res[mode]['hit_rate']:.3f}")
    for L in layers:
        L.destroy()
    moe.moe_set_cache_bytes(moe.SIZE_MAX)
    moe.moe_set_cache_policy(moe.MOE_CACHE_LRU)
    causal = [m for m in res if not m.endswith("+trace")] or list(res)
    best = max(causal, key=lambda m: res[m]["tokens_per_s"])
    b = res[best]
    return {"metric": "moe_streaming_decode_tokens_per_s", "value": b["tokens_per_s"], "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": warmup, "ms_per_step": b["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_DECODE,
            "data": "synthetic", "config": config_json(cfg, args) | {"mode": best},
            "roofline": {"bound": "h2d", "achieved": b["h2d_gbs"], "peak": h2d_peak, "unit": "GB/s",
                         "frac": b["h2d_frac"], "traffic": None,
                         "peak_source": "pinned cudaMemcpyAsync H2D probe, 256 MiB, best of 10"},
            "cache": {"slots": cfg.cache_bytes // layers[0].expert_bytes, "modes": res},
            "gpu_launches": b["gpu_launches"], "clocks": b["clocks"]}


def h2d_probe(dev) -> float:
    import torch
    src = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(10):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        dst.copy_(src, non_blocking=True)
        e.record()
        torch.cuda.synchronize()
        best = max(best, src.numel() / (s.elapsed_time(e) / 1e3) / 1e9)
    return best


# ----------------------------------------------------------------------------- distributed plumbing
_PG = None


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, dev) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1, choices=[1, 2, 3, 4])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--clocks-dir", default=tempfile.gettempdir(),
                    help="where the raw nvidia-smi samples of the timed region are written")
    ap.add_argument("--stream-modes", default="",
                    help="config 4: comma-separated modes out of " + ",".join(STREAM_MODES + EXTRA_STREAM_MODES) +
                         " (default: " + ",".join(STREAM_MODES) + ")")
    ap.add_argument("--no-extra", action="store_true",
                    help="config 1 only: skip the batched-decode and prefill lines added to the JSON")
    ap.add_argument("--small", action="store_true",
                    help="32 routed experts instead of 256 (same per-launch work at T=1; for ncu captures)")
    args = ap.parse_args()
    cfg = synth.WORKLOADS[args.config]
    if args.small:
        import dataclasses
        cfg = dataclasses.replace(cfg, n_experts=32, name=cfg.name + " [32 experts]")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, cfg)), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    res = run_ours(args, cfg, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on this host's cores (one process per core), with the
        # one-core figure beside it; configs 3 and 4 take config-1 tokens (the
        # oracle's cost per token is the same per expert)
        idx = args.config if args.config in (1, 2) else 1
        res["cpu_baseline"] = oracle_all_cores(idx, budget_s=15.0)
        res["cpu_baseline_1core"] = oracle_sample_rate(idx, n_tokens=3, budget_s=10.0)
        if idx != args.config:
            for k in ("cpu_baseline", "cpu_baseline_1core"):
                res[k]["sample"] += "; decode tokens of the config-1 layer (same per-expert cost)"
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
