"""Parity at the full workload sizes, in the launch configuration bench.py
times: dsa_forward over the whole batch, inputs from the seeded device
generator with the seed bench.py's rank 0 uses.

Two kinds of check on each workload's one run:
  * every row, on the device: the kept index list has min(2048, n_vis)
    entries, strictly ascending, inside [0, n_vis), -1 padded; o_lat and lse
    are finite (no oracle needed);
  * rows checked against the oracle one by one: every row of the decode
    workloads (4, 64 and 32 rows), 256 rows of each prefill workload (rows 0,
    1, 2047, 2048 and the last, the rest a seeded sample).  For each: indexer
    scores (materialised path) within 2e-2 * max|I|, the kept set equal to the
    oracle's up to pairs inside the 1e-3 * max|I| tie band, attention on the
    GPU's index set within max-abs 2e-2 / rel-L2 5e-3 (lse too), and recall
    of every surviving planted position.
The oracle rows are split into shards so that no single test runs long.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import workloads as wl

from gpu_util import (SCALE, assert_attention_close, assert_scores_close, assert_selection_ok, host_rows,
                      host_selected_rows)

pytestmark = pytest.mark.gpu

FIXED_PREFILL_ROWS = (0, 1, 2047, 2048)
PREFILL_SAMPLE = 256


def oracle_rows(cfg, T):
    """Rows checked against the oracle: all of a decode batch, 256 of a prefill."""
    if wl.WORKLOADS[cfg]["kind"] == "decode":
        return list(range(T))
    fixed = sorted(set(FIXED_PREFILL_ROWS) | {T - 1})
    rest = np.setdiff1d(np.arange(T), fixed)
    pick = np.random.default_rng(20241).choice(rest, PREFILL_SAMPLE - len(fixed), replace=False)
    return sorted(fixed + [int(x) for x in pick])


# (cfg, number of oracle shards); rows per shard stay at most 64
SHARDS = {0: 1, 1: 4, 3: 2, 2: 4, 4: 8}
PLAN = [(cfg, s) for cfg in (0, 1, 3, 2, 4) for s in ["every-row"] + list(range(SHARDS[cfg]))]

_RUN = {}


def _forward(cfg):
    """dsa_forward on workload `cfg` at full size (cached for that workload's tests)."""
    import torch
    if _RUN.get("cfg") == cfg:
        return _RUN
    _RUN.clear()
    torch.cuda.empty_cache()
    from indexer_selected_sparse_dsa_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    c = wl.make_workload_torch(cfg, dev, seed=cfg)            # same seed as bench.py rank 0
    T, k = c.T, wl.TOPK
    max_n = int(c.n_vis.max().item())
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((T, 64), float("nan"), dtype=torch.float32, device=dev)
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    ws = B.workspace(B.DSA_OP_FORWARD, T, max_n, k, device=dev)
    B.dsa_forward(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, max_n, k, wl.SCALE, o, lse, idx, ws)
    B.dsa_sync_status()
    _RUN.update(cfg=cfg, c=c, o=o, lse=lse, idx=idx, ws=ws, max_n=max_n, k=k)
    return _RUN


def _check_every_row(run):
    import torch
    c, idx, k = run["c"], run["idx"], run["k"]
    nv = c.n_vis.to(torch.int64)[:, None]
    K = torch.clamp(nv, max=k)
    j = torch.arange(k, device=idx.device)[None, :]
    x = idx.to(torch.int64)
    inside = j < K
    bad_kept = inside & ((x < 0) | (x >= nv))
    bad_pad = (~inside) & (x != -1)
    bad_order = (j[:, 1:] < K) & (x[:, 1:] <= x[:, :-1])
    rows_bad = bad_kept.any(1) | bad_pad.any(1) | bad_order.any(1)
    nbad = int(rows_bad.sum().item())
    assert nbad == 0, f"{nbad} rows hold an invalid index list, first {int(torch.nonzero(rows_bad)[0].item())}"
    assert bool(torch.isfinite(run["o"]).all().item()), "non-finite o_lat"
    lse_ok = torch.isfinite(run["lse"]) | (run["lse"] == -float("inf"))
    assert bool(lse_ok.all().item()), "NaN lse"


@pytest.mark.parametrize("cfg,shard", PLAN, ids=[f"w{c}-{s}" for c, s in PLAN])
def test_full_size_workload(cfg, shard):
    import torch
    run = _forward(cfg)
    c, k, T = run["c"], run["k"], run["c"].T
    if shard == "every-row":
        _check_every_row(run)
        return
    rows_all = oracle_rows(cfg, T)
    rows = list(np.array_split(np.asarray(rows_all), SHARDS[cfg])[shard])
    rows = [int(r) for r in rows]
    streams = run["ws"].numel() < T * run["max_n"] * 4 // 8
    # indexer side: the oracle's fp64 scores of these rows over their own prefixes
    for b0 in range(0, len(rows), 16):
        rb = rows[b0:b0 + 16]
        h = host_rows(c, rb, with_kv=False)
        S_ref = oracle.indexer_scores(h["q_I"], h["w"], h["k_I"], h["kv_start"], h["n_vis"],
                                      score_ld=int(h["n_vis"].max()))
        if not streams:
            # the score matrix dsa_forward materialised sits after the plan in the workspace
            ld = (run["max_n"] + 3) // 4 * 4
            plan_bytes = B.dsa_workspace_size(B.DSA_OP_INDEXER, T, run["max_n"], k)
            scores = run["ws"][plan_bytes:plan_bytes + T * ld * 4].view(torch.float32).view(T, ld)
            assert_scores_close(scores[rb].cpu().numpy(), S_ref, h["n_vis"])
        else:
            # the chunked prefill streams its scores (32 GB as a matrix): no score matrix in the workspace
            assert cfg == 4
        g_idx = run["idx"][rb].cpu().numpy()
        assert_selection_ok(g_idx, S_ref, h["n_vis"], k, rows=rb)
        for j, r in enumerate(rb):
            p = h["plants"][j][h["plants"][j] >= 0]
            assert np.isin(p, g_idx[j]).all(), f"row {r}: planted position dropped"
        # attention side: the oracle on the GPU's index set
        a = host_selected_rows(c, rb, g_idx)
        o_ref, lse_ref = oracle.sparse_mla(a["q"], a["kv"], a["kv_start"], a["idx"], SCALE)
        assert_attention_close(run["o"][rb].cpu().numpy(), run["lse"][rb].cpu().numpy(), o_ref, lse_ref)



# Block-level variant at the bench's size (bench.py --block-sparse: the 64-row, 128K
# decode workload; 1024 blocks per row, 64 anchor blocks, 16 dynamic blocks): the
# block choice on three rows equals the oracle's choice on the GPU's own fp32
# scores, and the fused output and the three branches' lse match the oracle run on
# those rows' own prefixes.
BLOCK_ROWS = (0, 31, 63)


def test_block_sparse_full_size_rows():
    import torch
    _RUN.clear()
    torch.cuda.empty_cache()
    from indexer_selected_sparse_dsa_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    c = wl.make_workload_torch(1, dev, seed=1)                 # same seed as bench.py rank 0
    T = c.T
    max_n = int(c.n_vis.max().item())
    r = np.random.default_rng(77)
    gates_h = r.uniform(0, 1, (T, 64, 3)).astype(np.float32)
    gates = torch.from_numpy(gates_h).to(dev)
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device=dev)
    lse = torch.full((3, T, 64), float("nan"), dtype=torch.float32, device=dev)
    blocks = torch.full((T, oracle.BLOCK_TOPK), -7, dtype=torch.int32, device=dev)
    ws = B.workspace(B.DSA_OP_BLOCK_SPARSE, T, max_n, 0, device=dev)
    B.dsa_block_sparse_attn(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, max_n, gates, SCALE, o, lse,
                            blocks, ws)
    B.dsa_sync_status()
    ld = (max_n + 3) // 4 * 4
    off = B.dsa_workspace_size(B.DSA_OP_INDEXER, T, max_n, 0)
    rows = list(BLOCK_ROWS)
    S_gpu = ws[off:off + T * ld * 4].view(torch.float32).view(T, ld)[rows].cpu().numpy()
    h = host_rows(c, rows)
    S_ref = oracle.indexer_scores(h["q_I"], h["w"], h["k_I"], h["kv_start"], h["n_vis"], score_ld=ld)
    assert_scores_close(S_gpu, S_ref, h["n_vis"])
    S_own = np.where(np.arange(ld)[None, :] < h["n_vis"][:, None], S_gpu, 0).astype(np.float64)
    loc, anc, dyn, blk = oracle.block_branch_sets(S_own, h["n_vis"])
    assert np.array_equal(blocks[rows].cpu().numpy(), blk), "block choice differs on the kernel's own scores"
    g = gates_h[rows].astype(np.float64)
    outs, lses = [], []
    for idxs in (loc, anc, dyn):
        o_b, lse_b = oracle.sparse_mla(h["q"], h["kv"], h["kv_start"], idxs, SCALE)
        outs.append(o_b)
        lses.append(lse_b)
    o_ref = sum(g[:, :, b, None] * outs[b] for b in range(3))
    lse_g = lse.cpu().numpy()
    assert_attention_close(o[rows].cpu().numpy(), lse_g[2][rows], o_ref, lses[2])
    for b in range(2):  # the local and anchor branches' lse
        d = np.abs(lse_g[b][rows] - lses[b])
        assert np.isfinite(lse_g[b][rows]).all() and d.max() <= 2e-2, (b, float(d.max()))


# NEXT rows at the bench's size (the 64-row, 128K decode workload), on the index
# set dsa_forward selects: a shared layer of an IndexShare group (bench.py
# --indexshare: its own queries and latent cache, the full layer's indices) and
# the dense + sparse layer (bench.py --dense-window 512), each checked against the
# oracle on three rows.
NEXT_ROWS = (0, 33, 63)


def test_indexshare_and_dense_sparse_full_size_rows():
    import torch
    run = _forward(1)
    c, idx, T, k = run["c"], run["idx"], run["c"].T, run["k"]
    dev = idx.device
    rows = list(NEXT_ROWS)
    g_idx = idx[rows].cpu().numpy()
    # shared layer: its own q and kv, the full layer's idx
    q1, kv1 = wl.make_shared_layer_torch(c, 1, dev, seed=1)
    o1 = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device=dev)
    l1 = torch.full((T, 64), float("nan"), dtype=torch.float32, device=dev)
    ws_a = B.workspace(B.DSA_OP_SPARSE_MLA, T, 0, k, device=dev)
    B.dsa_sparse_mla_attn(q1, kv1, c.kv_start, idx, SCALE, o1, l1, ws_a)
    B.dsa_sync_status()
    c1 = dataclasses.replace(c, q=q1, kv=kv1)
    a = host_selected_rows(c1, rows, g_idx)
    o_ref, lse_ref = oracle.sparse_mla(a["q"], a["kv"], a["kv_start"], a["idx"], SCALE)
    assert_attention_close(o1[rows].cpu().numpy(), l1[rows].cpu().numpy(), o_ref, lse_ref)
    del q1, kv1, c1
    # dense + sparse: the last 512 visible positions and the selected set, fused per (row, head)
    W = 512
    gate_h = np.random.default_rng(78).uniform(0, 1, (T, 64)).astype(np.float32)
    gate = torch.from_numpy(gate_h).to(dev)
    o2 = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device=dev)
    ld2 = torch.full((T, 64), float("nan"), dtype=torch.float32, device=dev)
    ls2 = torch.full((T, 64), float("nan"), dtype=torch.float32, device=dev)
    ws_d = B.workspace(B.DSA_OP_DENSE_SPARSE, T, 0, k, device=dev)
    B.dsa_dense_sparse_attn(c.q, c.kv, c.kv_start, c.n_vis, idx, W, gate, SCALE, o2, ld2, ls2, ws_d)
    B.dsa_sync_status()
    h = host_rows(c, rows)
    o_ref2, lsed_ref, lses_ref = oracle.dense_sparse(h["q"], h["kv"], h["kv_start"], h["n_vis"], g_idx, W,
                                                     gate_h[rows], SCALE)
    assert_attention_close(o2[rows].cpu().numpy(), ls2[rows].cpu().numpy(), o_ref2, lses_ref)
    d = np.abs(ld2[rows].cpu().numpy() - lsed_ref)
    assert d.max() <= 2e-2, float(d.max())
