"""The streaming cache's replacement policies on the expert-streaming routing
trace, simulated on the host with the same model the GPU tests check the
library against (CPU only)."""
import dataclasses

import pytest

from routed_expert_ffn_forward_b200 import synth
from tests.cache_model import CacheModel


def replay(policy, slots, steps):
    cfg = dataclasses.replace(synth.STREAMING, steps=steps)
    trace = synth.streaming_trace(cfg)
    m = CacheModel(slots, policy)
    for s in range(steps):
        for l in range(cfg.n_layers):
            m.forward(l, trace[s, l].tolist() + [cfg.n_experts + j for j in range(cfg.n_shared)])
    return m


def test_lru_basic_eviction_order():
    m = CacheModel(2, "lru")
    m.forward(0, [1])
    m.forward(0, [2])
    m.forward(0, [3])          # evicts expert 1, the least recently used
    assert (0, 1) not in m.key and (0, 2) in m.key and m.evictions == 1


def test_lfu_keeps_the_frequent_expert():
    m = CacheModel(3, "lfu")
    for e in (1, 9, 1, 9, 1):      # expert 1 enters use three times, expert 9 twice
        m.forward(0, [e])
    m.forward(0, [2])
    m.forward(0, [3])              # expert 2 was used by the previous forward: evict 9
    assert (0, 1) in m.key and (0, 2) in m.key and (0, 9) not in m.key
    assert m.use[(0, 1)][0] == 3


def test_lfu_counts_arrivals_not_repeats():
    m = CacheModel(2, "lfu")
    for _ in range(5):
        m.forward(0, [1])          # used by five forwards in a row: one arrival
    assert m.use[(0, 1)][0] == 1
    m.forward(0, [2])
    m.forward(0, [1])              # back after a gap: a second arrival
    assert m.use[(0, 1)][0] == 2


def test_lfu_counts_age():
    m = CacheModel(1, "lfu")
    for i in range(CacheModel.AGE_EVERY):
        m.forward(0, [i % 2])      # every forward is an arrival
    assert m.arrivals == CacheModel.AGE_EVERY
    assert m.use[(0, 0)][0] == (CacheModel.AGE_EVERY // 2) // 2 and m.use[(0, 1)][0] == 16


@pytest.mark.slow
def test_lfu_beats_lru_on_the_streaming_trace():
    # 8 layers, Zipf(1.1) popularity, 60 % of experts kept step to step,
    # 484 slots: frequency keeps the popular experts that recency loses
    lru, lfu = replay("lru", 484, 300), replay("lfu", 484, 300)
    rate = lambda m: m.hits / (m.hits + m.misses)
    assert rate(lfu) > rate(lru) + 0.01, (rate(lru), rate(lfu))
    assert lfu.misses < 0.92 * lru.misses
