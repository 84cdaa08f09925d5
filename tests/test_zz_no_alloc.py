"""The allocation-free indexer entry point, dsa_indexer_scores_noalloc.

It exists for callers that are not allowed to allocate device memory: code
running inside a framework that owns every byte of GPU memory and plans its
pool once at start-up, or a plug-in that is handed tensors but no allocator.
Instead of a caller-provided workspace it keeps its scratch (the query-tile
plan) in a fixed array inside the library.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import build
from indexer_selected_sparse_dsa_b200 import workloads as wl


def _case(seed, seq_lens, queries):
    return wl.make_case_numpy(seq_lens, queries, seed=seed, n_plant=4)


def _dev(c):
    import torch

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    return (bf(c.q_I), bf(c.w), bf(c.k_I), torch.from_numpy(c.kv_start).cuda(), torch.from_numpy(c.n_vis).cuda())


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    """Two consecutive calls (different shapes, so the second overwrites the
    first one's plan in the shared array) agree with dsa_indexer_scores."""
    import torch
    build.build()
    cases = [
        _case(101, [900, 300], [(0, 900), (0, 899), (0, 640), (1, 300), (1, 17), (0, 1)]),
        _case(102, [2000], [(0, t + 1) for t in range(0, 2000, 9)]),
    ]
    for c in cases:
        q_I, w, k_I, ks, nv = _dev(c)
        T = c.T
        ld = (int(c.n_vis.max()) + 3) // 4 * 4
        ref = torch.full((T, ld), float("nan"), device="cuda")
        ws = B.workspace(B.DSA_OP_INDEXER, T, ld, 0)
        B.dsa_indexer_scores(q_I, w, k_I, ks, nv, ref, ws)
        got = torch.full((T, ld), float("nan"), device="cuda")
        B.dsa_indexer_scores_noalloc(q_I, w, k_I, ks, nv, got)
        B.dsa_sync_status()
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        o = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, ld)
        for i, n in enumerate(c.n_vis):
            tol = 2e-2 * np.max(np.abs(o[i, :n]))          # the indexer parity tolerance
            assert np.max(np.abs(g[i, :n] - r[i, :n])) <= tol
            assert np.max(np.abs(g[i, :n] - o[i, :n])) <= tol   # and against the oracle directly
            assert np.isnan(g[i, n:]).all()


@pytest.mark.gpu
def test_noalloc_at_its_row_limit_fills_the_scratch_plan():
    """DSA_NOALLOC_MAX_ROWS query rows, each over a sequence of its own (no two
    rows share a query tile), so the plan uses every entry of the fixed array."""
    import torch
    build.build()
    T = B.NOALLOC_MAX_ROWS
    rng = np.random.default_rng(103)
    lens = 1 + (np.arange(T) * 97) % 200                   # 1 .. 200 keys per sequence
    starts = np.zeros(T, np.int64)
    starts[1:] = np.cumsum(lens)[:-1]
    L = int(lens.sum())
    q_I = wl.bf16_from_f32(rng.standard_normal((T, 32, 128), dtype=np.float32) / np.float32(np.sqrt(128)))
    w = wl.bf16_from_f32(rng.random((T, 32), dtype=np.float32))
    k_I = wl.bf16_from_f32(rng.standard_normal((L, 128), dtype=np.float32) / np.float32(np.sqrt(128)))
    n_vis = lens.astype(np.int32)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    ld = 200
    ks, nv = torch.from_numpy(starts).cuda(), torch.from_numpy(n_vis).cuda()
    got = torch.full((T, ld), float("nan"), device="cuda")
    B.dsa_indexer_scores_noalloc(bf(q_I), bf(w), bf(k_I), ks, nv, got)
    B.dsa_sync_status()
    ref = torch.full((T, ld), float("nan"), device="cuda")
    B.dsa_indexer_scores(bf(q_I), bf(w), bf(k_I), ks, nv, ref, B.workspace(B.DSA_OP_INDEXER, T, ld, 0))
    B.dsa_sync_status()
    g, r = got.cpu().numpy(), ref.cpu().numpy()
    o = oracle.indexer_scores(q_I, w, k_I, starts, n_vis, ld)
    for i in range(T):
        n = int(n_vis[i])
        tol = 2e-2 * np.max(np.abs(o[i, :n]))
        assert np.max(np.abs(g[i, :n] - o[i, :n])) <= tol, f"row {i}"
        assert np.max(np.abs(g[i, :n] - r[i, :n])) <= tol, f"row {i}"
        assert np.isnan(g[i, n:]).all(), f"row {i}: wrote past n_vis"


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    build.build()
    L = B.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = L.dsa_indexer_scores_noalloc(fake, fake, fake, 100, fake, fake, B.NOALLOC_MAX_ROWS + 1, fake, 8,
                                      ctypes.c_void_p(0))
    assert rc == B.DSA_ERR_INVALID_ARG
    assert "at most" in B.last_error()
