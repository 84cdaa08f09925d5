"""fp64 CPU oracle for the DSA sparse-attention step — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The library path never does.

Thin numpy front end over ``dsa_oracle.cpp`` (plain C++, fp64, std::thread
over query rows).  ``build()`` compiles it with g++; ``lib()`` builds on first
use when the shared object is missing or stale.

Functions (all inputs are bf16 bit patterns as uint16 arrays):
  indexer_scores(q_I, w, k_I, kv_start, n_vis, score_ld) -> float64 [T, score_ld]
  topk(scores, n_vis, topk)                              -> int32 [T, topk]
  sparse_mla(q, kv, kv_start, idx, scale)                -> (o_lat f64 [T,64,512], lse f64 [T,64])
  forward(case or arrays, topk, scale)                   -> (o_lat, lse, idx)
  dense_sparse(q, kv, kv_start, n_vis, idx, window, gate, scale)
                                                         -> (o_lat, lse_dense, lse_sparse)
  block_sparse(q_I, w, k_I, q, kv, kv_start, n_vis, gates, scale)
                                                         -> (o_lat, (lse x 3), branch sets)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")
# A test may point the front end at another build of the same source (the
# mutation test builds deliberately broken copies to show the pins catch them).
_SO_OVERRIDE = os.environ.get("DSA_ORACLE_SO")
_lib = None

NTHREADS = os.cpu_count() or 1


def build(force: bool = False) -> str:
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", _SRC, "-o", _SO + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(_SO + ".tmp", _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        if _SO_OVERRIDE:
            L = ctypes.CDLL(_SO_OVERRIDE)
        else:
            build()
            L = ctypes.CDLL(_SO)
        P = ctypes.c_void_p
        L.oracle_indexer_scores.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int64, P, ctypes.c_int]
        L.oracle_topk.argtypes = [P, ctypes.c_int64, P, ctypes.c_int, ctypes.c_int, P, ctypes.c_int]
        L.oracle_sparse_mla.argtypes = [P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P, ctypes.c_int]
        L.oracle_forward.argtypes = [P, P, P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_double, P, P, P, ctypes.c_int]
        L.oracle_dims.argtypes = [P]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def dims():
    out = np.zeros(6, np.int32)
    lib().oracle_dims(_p(out))
    return tuple(int(x) for x in out)


def indexer_scores(q_I, w, k_I, kv_start, n_vis, score_ld=None, nthreads=NTHREADS):
    q_I, w, k_I = _c(q_I, np.uint16), _c(w, np.uint16), _c(k_I, np.uint16)
    kv_start, n_vis = _c(kv_start, np.int64), _c(n_vis, np.int32)
    T = n_vis.shape[0]
    if score_ld is None:
        score_ld = int(n_vis.max()) if T else 1
    out = np.full((T, score_ld), np.nan, np.float64)
    lib().oracle_indexer_scores(_p(q_I), _p(w), _p(k_I), _p(kv_start), _p(n_vis), T, score_ld, _p(out), nthreads)
    return out


def topk(scores, n_vis, k, nthreads=NTHREADS):
    scores = _c(scores, np.float64)
    n_vis = _c(n_vis, np.int32)
    T = n_vis.shape[0]
    idx = np.empty((T, k), np.int32)
    lib().oracle_topk(_p(scores), scores.shape[1], _p(n_vis), T, k, _p(idx), nthreads)
    return idx


def sparse_mla(q, kv, kv_start, idx, scale, nthreads=NTHREADS):
    q, kv = _c(q, np.uint16), _c(kv, np.uint16)
    kv_start, idx = _c(kv_start, np.int64), _c(idx, np.int32)
    T, k = idx.shape
    o = np.empty((T, 64, 512), np.float64)
    lse = np.empty((T, 64), np.float64)
    lib().oracle_sparse_mla(_p(q), _p(kv), _p(kv_start), _p(idx), T, k, float(scale), _p(o), _p(lse), nthreads)
    return o, lse


def forward(q_I, w, k_I, q, kv, kv_start, n_vis, k, scale, nthreads=NTHREADS):
    q_I, w, k_I = _c(q_I, np.uint16), _c(w, np.uint16), _c(k_I, np.uint16)
    q, kv = _c(q, np.uint16), _c(kv, np.uint16)
    kv_start, n_vis = _c(kv_start, np.int64), _c(n_vis, np.int32)
    T = n_vis.shape[0]
    o = np.empty((T, 64, 512), np.float64)
    lse = np.empty((T, 64), np.float64)
    idx = np.empty((T, k), np.int32)
    lib().oracle_forward(_p(q_I), _p(w), _p(k_I), _p(q), _p(kv), _p(kv_start), _p(n_vis), T, k,
                         float(scale), _p(o), _p(lse), _p(idx), nthreads)
    return o, lse, idx


def window_indices(n_vis, window):
    """The dense branch's positions: n - window .. n - 1 of each row, -1 where
    negative (rows shorter than the window)."""
    n = np.asarray(n_vis, np.int64)[:, None]
    p = n - window + np.arange(window, dtype=np.int64)[None, :]
    return np.where(p >= 0, p, -1).astype(np.int32)


def dense_sparse(q, kv, kv_start, n_vis, idx, window, gate, scale, nthreads=NTHREADS):
    """Dense + sparse DSA layer ("GLM-5.2's DSA architecture: how dense and sparse
    attention split the work", section "DSA's core design"): local dense
    attention over the last ``window`` visible positions and sparse attention over
    ``idx``, fused per (row, head) with the caller's weight ``gate`` [T, 64]:
    o = gate * o_dense + (1 - gate) * o_sparse.  Each branch is ``sparse_mla``."""
    o_s, lse_s = sparse_mla(q, kv, kv_start, idx, scale, nthreads)
    o_d, lse_d = sparse_mla(q, kv, kv_start, window_indices(n_vis, window), scale, nthreads)
    g = np.asarray(gate, np.float64)[:, :, None]
    return g * o_d + (1.0 - g) * o_s, lse_d, lse_s


def forward_case(c, scale, nthreads=NTHREADS):
    return forward(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, c.topk, scale, nthreads)


# ---------------------------------------------------------------------------
# Block-level variant ("GLM-5: 744B parameters, 202K long context", section 2,
# "Decoupled Sparse Attention"): the context is cut into 128-token blocks and
# three branches attend, each over its own set of positions, and are fused with
# weights: a local branch (the query's block and its neighbours, 3 x 128 = 384
# positions, the later one masked by causality), a global anchor branch (one
# block in every 16) and a dynamic branch (each query's 16 most relevant
# blocks).  The page does not say how a block's relevance is scored: read here
# as the largest lightning-indexer score among the block's visible positions,
# the 16 best blocks kept under (score descending, block ascending).  The
# page's fusion weights are learned; here they are the caller's gates
# [T, 64, 3] (local, anchor, dynamic).
# ---------------------------------------------------------------------------

BLOCK = 128         # tokens per block
BLOCK_TOPK = 16     # dynamic branch: blocks per query
ANCHOR_EVERY = 16   # one anchor block in every 16 blocks
LOCAL_SIDE = 1      # local branch: neighbour blocks on each side of the query's block


def block_scores(scores, n_vis):
    """Per row, the score of each visible block: the largest score among its
    visible positions.  Returns a list of float arrays (one per row)."""
    out = []
    for i, n in enumerate(np.asarray(n_vis)):
        n = int(n)
        nb = (n + BLOCK - 1) // BLOCK
        out.append(np.array([np.max(scores[i, b * BLOCK:min((b + 1) * BLOCK, n)]) for b in range(nb)]))
    return out


def block_branch_sets(scores, n_vis):
    """Index lists of the three branches, ascending, -1 padded:
    local [T, 3*128], anchor [T, ceil(max blocks / 16) * 128], dynamic [T, 16*128],
    and the dynamic branch's blocks [T, 16]."""
    n_vis = np.asarray(n_vis)
    T = n_vis.shape[0]
    max_nb = int((int(n_vis.max()) + BLOCK - 1) // BLOCK) if T else 1
    W_loc = (2 * LOCAL_SIDE + 1) * BLOCK
    W_anc = ((max_nb + ANCHOR_EVERY - 1) // ANCHOR_EVERY) * BLOCK
    W_dyn = BLOCK_TOPK * BLOCK
    loc = np.full((T, W_loc), -1, np.int32)
    anc = np.full((T, W_anc), -1, np.int32)
    dyn = np.full((T, W_dyn), -1, np.int32)
    blk = np.full((T, BLOCK_TOPK), -1, np.int32)
    bsc = block_scores(scores, n_vis)
    for i, n in enumerate(n_vis):
        t = int(n) - 1
        qb = t // BLOCK
        lo = max(0, (qb - LOCAL_SIDE) * BLOCK)
        p = np.arange(lo, t + 1)
        loc[i, :p.size] = p
        p = np.concatenate([np.arange(b * BLOCK, min(b * BLOCK + BLOCK, t + 1)) for b in range(0, qb + 1, ANCHOR_EVERY)])
        anc[i, :p.size] = p
        order = sorted(range(qb + 1), key=lambda b: (-bsc[i][b], b))[:BLOCK_TOPK]
        kept = sorted(order)
        blk[i, :len(kept)] = kept
        p = np.concatenate([np.arange(b * BLOCK, min(b * BLOCK + BLOCK, t + 1)) for b in kept])
        dyn[i, :p.size] = p
    return loc, anc, dyn, blk


def block_sparse(q_I, w, k_I, q, kv, kv_start, n_vis, gates, scale, nthreads=NTHREADS):
    """The block-level layer: indexer scores, the three branches' sets, one
    latent attention per branch (``sparse_mla``), fused per (row, head):
    o = sum_b gates[:, :, b] * o_b (b = local, anchor, dynamic).
    Returns (o_lat, (lse_local, lse_anchor, lse_dynamic), sets)."""
    S = indexer_scores(q_I, w, k_I, kv_start, n_vis, nthreads=nthreads)
    sets = block_branch_sets(S, n_vis)
    outs, lses = [], []
    for idx in sets[:3]:
        o_b, lse_b = sparse_mla(q, kv, kv_start, idx, scale, nthreads)
        outs.append(o_b)
        lses.append(lse_b)
    g = np.asarray(gates, np.float64)
    o = sum(g[:, :, b, None] * outs[b] for b in range(3))
    return o, tuple(lses), sets
