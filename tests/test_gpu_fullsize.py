"""Parity at the full workload sizes, in the launch configuration bench.py
times (dsa_forward on the whole batch, inputs from the seeded device
generator), checked on sampled rows the oracle computes one by one:
indexer scores, validity of the kept set under the tie band, attention on the
GPU's index set, and recall of every surviving planted position."""
import numpy as np
import pytest

import oracle
from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import workloads as wl

from gpu_util import SCALE, assert_attention_close, assert_scores_close, assert_selection_ok, host_rows

pytestmark = pytest.mark.gpu

SAMPLES = {
    0: [0, 1, 2, 3],
    1: [0, 31, 63],
    2: [0, 1, 2047, 2048, 20000, 32767],
    3: [0, 1, 30, 31],
    4: [0, 4095, 8191],
}


@pytest.mark.parametrize("cfg", [0, 1, 3, 2, 4])
def test_full_size_workload_sampled_rows(cfg):
    import torch
    from indexer_selected_sparse_dsa_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    c = wl.make_workload_torch(cfg, dev, seed=cfg)            # same seed as bench.py rank 0
    T, k = c.T, wl.TOPK
    max_n = int(c.n_vis.max().item())
    o = torch.empty((T, 64, 512), dtype=torch.float32, device=dev)
    lse = torch.empty((T, 64), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    ws = B.workspace(B.DSA_OP_FORWARD, T, max_n, k, device=dev)
    B.dsa_forward(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, max_n, k, wl.SCALE, o, lse, idx, ws)
    B.dsa_sync_status()
    rows = SAMPLES[cfg]
    h = host_rows(c, rows)
    S_ref = oracle.indexer_scores(h["q_I"], h["w"], h["k_I"], h["kv_start"], h["n_vis"],
                                  score_ld=int(h["n_vis"].max()))
    if cfg != 4:
        # the score matrix dsa_forward materialised sits after the plan in the workspace
        ld = (max_n + 3) // 4 * 4
        plan_bytes = B.dsa_workspace_size(B.DSA_OP_INDEXER, T, max_n, k)
        scores = ws[plan_bytes:plan_bytes + T * ld * 4].view(torch.float32).view(T, ld)
        assert_scores_close(scores[rows].cpu().numpy(), S_ref, h["n_vis"])
    else:
        # the chunked prefill streams its scores (32 GB as a matrix): the workspace holds no score matrix
        assert ws.numel() < T * max_n * 4 // 8
    g_idx = idx[rows].cpu().numpy()
    assert_selection_ok(g_idx, S_ref, h["n_vis"], k)
    o_ref, lse_ref = oracle.sparse_mla(h["q"], h["kv"], h["kv_start"], g_idx, SCALE)
    assert_attention_close(o[rows].cpu().numpy(), lse[rows].cpu().numpy(), o_ref, lse_ref)
    for j, r in enumerate(rows):
        p = h["plants"][j][h["plants"][j] >= 0]
        assert np.isin(p, g_idx[j]).all(), f"row {r}: planted position dropped"
