"""The bench's algorithmic work per step (the roofline numerators) against the
closed forms of the method's shapes: 32 indexer heads x 128 dims per (query,
visible key) pair, 2048 selected positions per query, 64 heads over 576-dim
keys and 512-dim values, 256 B per key of the indexer cache and 1152 B per
latent row ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
section 2.1 table and section 2.2)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from indexer_selected_sparse_dsa_b200 import workloads as wl  # noqa: E402


def _rows(cfg):
    seq_lens, queries, _ = wl.workload_layout(cfg)
    starts = np.concatenate([[0], np.cumsum(seq_lens)[:-1]]).astype(np.int64)
    n_vis = np.array([n for _, n in queries], np.int32)
    kv_start = np.array([starts[s] for s, _ in queries], np.int64)
    return n_vis, kv_start


def test_decode_128k_step_work():
    n_vis, kv_start = _rows(1)
    m = bench.work_model(n_vis, kv_start)
    T, n, k = 64, 131072, 2048
    assert m["indexer_flops"] == 2 * 32 * 128 * n * T                   # 68.7 GFLOP
    assert m["attention_flops"] == 2 * 64 * k * (576 + 512) * T          # 18.3 GFLOP
    keys = 256 * n * T                                                  # every key row once
    gathered = 1152 * k * T                                             # every selected latent row once
    io = T * (32 * 128 * 2 + 32 * 2 + 64 * 576 * 2 + 64 * 512 * 4 + 64 * 4)
    assert m["step_bytes"] == keys + gathered + io                      # 2.30 GB
    assert abs(m["step_bytes"] / 1e9 - 2.31) < 0.01


def test_shared_cache_keys_count_once():
    n_vis, kv_start = _rows(0)             # 4 queries over one 32K cache
    m = bench.work_model(n_vis, kv_start)
    assert np.all(kv_start == kv_start[0])
    assert m["indexer_bytes"] == 256 * 32768 + (4 * 32768 + 32 * 128 * 2 + 32 * 2) * 4


def test_prefill_32k_flops():
    n_vis, kv_start = _rows(2)
    m = bench.work_model(n_vis, kv_start)
    N = 32768
    pairs = N * (N + 1) // 2                                            # causal (query, key) pairs
    assert m["indexer_flops"] == 2 * 32 * 128 * pairs                   # 4.40 TFLOP
    sel = 2048 * 2049 // 2 + 2048 * (N - 2048)                          # min(2048, t + 1) summed
    assert m["attention_flops"] == 2 * 64 * (576 + 512) * sel           # 9.05 TFLOP
    assert abs(m["indexer_flops"] / 1e12 - 4.40) < 0.01 and abs(m["attention_flops"] / 1e12 - 9.05) < 0.01


def test_chunked_prefill_1m_flops():
    n_vis, kv_start = _rows(4)
    m = bench.work_model(n_vis, kv_start)
    prefix, new = 1040384, 8192
    pairs = new * prefix + new * (new + 1) // 2
    assert m["indexer_flops"] == 2 * 32 * 128 * pairs                   # 70.1 TFLOP
    assert abs(m["indexer_flops"] / 1e12 - 70.1) < 0.05
