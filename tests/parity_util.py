"""Comparison rules between the CUDA path and the CPU oracle.

Tolerances (the layer's stated bar):
  * router indices: the GPU's id set equals the oracle's for every token whose
    oracle top-k gap l_(k) - l_(k+1) is at least 1e-4; a token inside that
    window may pick either side of the tie, and its GPU set must then be a valid
    top-k within 1e-4 (every picked logit >= l_(k) - 1e-4);
  * outputs: max|out - ref| <= 2e-2 * max|ref| and
    sum|out - ref| / sum|ref| <= 2e-3 (L1-relative "mean relative error"),
    where ref is the oracle's output rounded to bf16 like the layer's output;
    near-tie tokens are compared with the oracle run on the GPU's ids.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_ref as ref

GAP = 1e-4
MAX_REL = 2e-2
MEAN_REL = 2e-3


def bf16_bits_to_f64(bits):
    return ref.bf16_to_f64(bits)


def check_ids(gpu_ids: np.ndarray, logits64: np.ndarray, k: int):
    """Returns (near_tie_token_mask).  Asserts the index rule."""
    gap = ref.topk_gap(logits64, k)
    want = ref.topk_ids(logits64, k)
    near = gap < GAP
    for t in range(len(gap)):
        g = np.sort(gpu_ids[t])
        if not near[t]:
            assert np.array_equal(g, np.sort(want[t])), f"token {t}: gpu {g} oracle {np.sort(want[t])}"
        else:
            kth = np.sort(logits64[t])[::-1][k - 1]
            assert len(set(g.tolist())) == k
            assert (logits64[t, g] >= kth - GAP).all(), f"token {t}: invalid near-tie pick {g}"
    return near


def output_errors(out_bits: np.ndarray, ref_bits: np.ndarray):
    o = bf16_bits_to_f64(out_bits)
    r = bf16_bits_to_f64(ref_bits)
    err = np.abs(o - r)
    max_rel = err.max() / max(np.abs(r).max(), 1e-300)
    mean_rel = err.sum() / max(np.abs(r).sum(), 1e-300)
    return max_rel, mean_rel


def check_outputs(out_bits: np.ndarray, ref_bits: np.ndarray, what: str = ""):
    assert np.isfinite(bf16_bits_to_f64(out_bits)).all(), f"{what}: non-finite output"
    max_rel, mean_rel = output_errors(out_bits, ref_bits)
    assert max_rel <= MAX_REL, f"{what}: max|err|/max|ref| = {max_rel:.3e}"
    assert mean_rel <= MEAN_REL, f"{what}: sum|err|/sum|ref| = {mean_rel:.3e}"
    return max_rel, mean_rel


# ------------------------------------------------------------------ oracle rows in parallel
def _oracle_rows_job(job):
    cfg, layer_index, x_bits, forced, tokens = job
    from threadpoolctl import threadpool_limits

    from routed_expert_ffn_forward_b200 import synth
    layer = dict(router_w=synth.router_weight(cfg, layer_index), router_b=synth.router_bias(cfg, layer_index),
                 experts=lambda e: synth.expert_tensors(cfg, layer_index, e))
    with threadpool_limits(limits=1):      # one core per process
        r = ref.moe_forward(x_bits, layer, cfg.top_k, cfg.gating, cfg.n_shared, cfg.inter, forced_ids=forced,
                            token_subset=tokens)
    return r["out_bf16"]


def oracle_rows(cfg, layer_index, x_bits, forced, tokens, workers=None):
    """The oracle's bf16 output rows for `tokens` (forced routing), computed by
    up to `workers` spawned processes, each over a share of the tokens (the
    oracle itself is unchanged; this only runs several of it at once)."""
    import multiprocessing as mp
    import os
    tokens = np.asarray(tokens)
    if workers is None:
        cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
        workers = max(1, min(16, cores, len(tokens)))
    chunks = [c for c in np.array_split(tokens, workers) if len(c)]
    if len(chunks) == 1:
        return _oracle_rows_job((cfg, layer_index, x_bits, forced, chunks[0]))
    with mp.get_context("spawn").Pool(len(chunks)) as pool:
        parts = pool.map(_oracle_rows_job, [(cfg, layer_index, x_bits, forced, c) for c in chunks])
    return np.concatenate(parts, axis=0)
