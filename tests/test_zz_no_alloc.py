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
        for i, n in enumerate(c.n_vis):
            tol = 2e-2 * np.max(np.abs(r[i, :n]))          # the indexer parity tolerance
            assert np.max(np.abs(g[i, :n] - r[i, :n])) <= tol
            assert np.isnan(g[i, n:]).all()


def test_noalloc_rejects_more_rows_than_its_scratch_holds():
    build.build()
    L = B.lib()
    fake = ctypes.c_void_p(1 << 20)
    rc = L.dsa_indexer_scores_noalloc(fake, fake, fake, 100, fake, fake, B.NOALLOC_MAX_ROWS + 1, fake, 8,
                                      ctypes.c_void_p(0))
    assert rc == B.DSA_ERR_INVALID_ARG
    assert "at most" in B.last_error()
