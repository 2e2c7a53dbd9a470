"""The benchmark's roofline arithmetic, checked on the CPU against the Q4_K
byte counts written out by hand (144 bytes per 256 weights)."""
import dataclasses
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from routed_expert_ffn_forward_b200 import synth  # noqa: E402


def test_decode_bytes_match_hand_count():
    cfg = synth.DECODE                      # H = 7168, I = 2048, k = 8, S = 1, T = 1
    ids = np.arange(8, dtype=np.int32)[None, :]
    gate = 2048 * (7168 // 256) * 144       # one gate (or up) matrix: 8,257,536 B
    down = 7168 * (2048 // 256) * 144       # 8,257,536 B
    assert gate == down == 8_257_536
    experts = 9                             # 8 routed + the shared one
    assert bench.algorithmic_bytes(cfg, ids, "gate_up") == experts * 2 * gate + 7168 * 2 + 9 * 2048 * 2
    assert bench.algorithmic_bytes(cfg, ids, "down") == experts * down + 9 * 2048 * 2 + 2 * 7168 * 2
    fwd = experts * (2 * gate + down) + 256 * 7168 * 4 + 2 * 7168 * 2
    assert bench.algorithmic_bytes(cfg, ids, "forward") == fwd
    assert abs(fwd - 230.3e6) < 0.1e6      # the per-token figure the layer is quoted on


def test_repeated_experts_counted_once():
    cfg = dataclasses.replace(synth.DECODE, tokens=3)
    ids = np.array([[0, 1, 2, 3, 4, 5, 6, 7]] * 3, dtype=np.int32)   # three tokens, same experts
    one = bench.algorithmic_bytes(cfg, ids[:1], "forward")
    three = bench.algorithmic_bytes(cfg, ids, "forward")
    assert three - one == 2 * 2 * 7168 * 2   # only x and out grow with the tokens


def test_few_row_gate_up_bytes():
    cfg = synth.BATCHED                     # T = 64: every expert has <= 64 rows (few-row tiles)
    ids = np.zeros((64, 8), dtype=np.int32)
    ids[:, 0] = 0                           # expert 0: 64 rows
    ids[:, 1:] = np.arange(1, 8)[None, :] + 7 * (np.arange(64)[:, None] % 4)
    ids[:60, 7] = 100 + np.arange(60) // 4  # 15 experts x 4 rows
    # columns 1-6: 24 experts x 16 rows; column 7 of the last 4 tokens: 4 experts x 1 row
    gate = 2048 * 28 * 144
    counts = np.bincount(ids.ravel(), minlength=256)
    assert np.all(np.sort(ids, axis=1)[:, 1:] != np.sort(ids, axis=1)[:, :-1])  # distinct picks per token
    assert int(np.sum(counts > 0)) == 44 and counts.max() == 64
    tiles, rows = 44 + 1, 64 * 9            # + the shared expert's 64 rows
    # the library's default at T = 64 is 64 rows: every tile is a few-row tile
    assert bench.tile_split(cfg, ids) == bench.tile_split(cfg, ids, few_rows=64) == (0, rows, tiles)
    # with 32, expert 0 and the shared expert (64 rows each) take the GEMM
    assert bench.tile_split(cfg, ids, few_rows=32) == (64 + 64, rows - 128, tiles - 2)
    expect = tiles * 2 * gate + rows * 7168 * 2 + rows * 2048 * 4
    assert bench.few_gate_up_bytes(cfg, ids) == expect
    assert bench.gate_up_gemm_flops(cfg, ids) == 0.0
    assert bench.few_rows_default(64) == 64 and bench.few_rows_default(4096) == 32


def test_prefill_flops():
    cfg = synth.PREFILL
    assert bench.flops(cfg, cfg.tokens) == 2.0 * 4096 * 9 * 3 * 7168 * 2048
    assert abs(bench.flops(cfg, cfg.tokens) - 3.247e12) < 0.001e12


def test_traffic_entry_tracks_its_source():
    """A recorded DRAM byte count is reported only while the kernel's source is
    the one it was captured from."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    for key, d in json.load(open(p)).items():
        src = os.path.join(ROOT, d["source"])
        current = hashlib.sha256(open(src, "rb").read()).hexdigest() == d["sha256"]
        got = bench.kernel_traffic(key)
        assert (got == float(d["bytes_per_launch"])) if current else got is None
    assert bench.kernel_traffic("config9:nothing") is None


def test_tile_split_hand_count():
    # 600 = 256+256+88 (GEMM), 300 = 256 | 44, 64 (few), 65 (GEMM), 1 (few),
    # 513 = 512 | 1, 320 = 256 | 64
    assert bench.split_rows([600, 300, 64, 65, 1, 513, 320], few_rows=64) == (600 + 256 + 65 + 512 + 256,
                                                                              44 + 64 + 1 + 1 + 64, 5)
    # the library's default, 32: 300 = 256 | 44 and 320 = 256 | 64 stay whole
    assert bench.split_rows([600, 300, 64, 65, 1, 513, 320]) == (600 + 300 + 64 + 65 + 512 + 320, 1 + 1, 2)
    assert bench.split_rows([600, 300, 64, 65, 1, 513, 320], few_rows=0) == (1863, 0, 0)
    assert bench.split_rows([256, 257], few_rows=1) == (256 + 256, 1, 1)


def test_gate_up_gemm_flops_hand_count():
    cfg = dataclasses.replace(synth.DECODE, tokens=70)
    # expert 0 on all 70 tokens (GEMM), experts 1..7 and the rest on few rows
    ids = np.array([[0] + [1 + (7 * t + j) % 200 for j in range(7)] for t in range(70)], dtype=np.int32)
    rows = 70 + 70                          # expert 0 and the shared expert
    assert bench.gate_up_gemm_flops(cfg, ids) == 2.0 * rows * 2 * 2048 * 7168


def test_tile_split_off_sends_everything_to_the_gemm():
    cfg = dataclasses.replace(synth.DECODE, tokens=6)
    ids = np.array([[0, 1] + [10 * j + t for j in range(1, 7)] for t in range(6)], dtype=np.int32)
    gemm, few, n_few = bench.tile_split(cfg, ids, few_rows=0)
    assert (gemm, few, n_few) == (6 * 8 + 6, 0, 0)


def test_oracle_all_cores_reports_its_workers():
    r = bench.oracle_all_cores(0, budget_s=0.2, max_workers=2)
    assert r["kind"] == "oracle" and r["unit"] == "tokens/s"
    assert 1 <= r["cores"] <= 2 and r["value"] > 0
    assert str(r["cores"]) in r["sample"]
