"""Pins for the fp64 oracle, each against something other than the oracle itself.

The pins are closed forms, algebraic identities that take a different route
through the arithmetic, textbook routines from scipy, brute force on tiny
inputs, and structural invariants stated on the pages:
  * "2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2 — the indexer only ranks,
    at most index_topk positions per query take part in attention;
  * "From a trillion dot products to two thousand: how DSA breaks N^2", "DSA full flow" — indexer over all history,
    top-2048, then softmax and V mix over those only;
  * same page, on the kept KV cache — unselected positions stay available to
    other queries (a shared cache is read, never consumed).
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from indexer_selected_sparse_dsa_b200 import workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))
rng0 = np.random.default_rng(1234)


def f32(b):
    return wl.bf16_to_f32(b).astype(np.float64)


def small_case(seed=0, L=300, T=5, n_plant=8, topk=64):
    queries = [(0, L - T + i + 1) for i in range(T)]
    c = wl.make_case_numpy([L], queries, seed, n_plant=n_plant, topk=topk)
    return c


def test_dims_match_config_table():
    # index_n_heads 32, index_head_dim 128, heads 64, kv_lora_rank 512, rope 64
    assert oracle.dims() == (32, 128, 64, 512, 64, 576)


# ----------------------------------------------------------------------------- indexer

def test_scores_collapsed_identity():
    """sum_h w_h (q_h . k) == (sum_h w_h q_h) . k  — computed here by the second route."""
    c = small_case(seed=1)
    S = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis)
    qf, wf, kf = f32(c.q_I), f32(c.w), f32(c.k_I)
    for i in range(c.T):
        v = (wf[i][:, None] * qf[i]).sum(axis=0)
        nv = c.n_vis[i]
        ref = kf[c.kv_start[i]:c.kv_start[i] + nv] @ v
        got = S[i, :nv]
        assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_scores_one_hot_head_exact():
    """w one-hot on head h reduces the score to one dot product; integer-valued
    bf16 inputs make every product and sum exact."""
    T, L = 3, 40
    r = np.random.default_rng(5)
    q = r.integers(-3, 4, size=(T, 32, 128)).astype(np.float32)
    k = r.integers(-3, 4, size=(L, 128)).astype(np.float32)
    for h in (0, 17, 31):
        w = np.zeros((T, 32), np.float32)
        w[:, h] = 1.0
        S = oracle.indexer_scores(wl.bf16_from_f32(q), wl.bf16_from_f32(w), wl.bf16_from_f32(k),
                                  np.zeros(T, np.int64), np.full(T, L, np.int32))
        for i in range(T):
            exact = [int(sum(int(a) * int(b) for a, b in zip(q[i, h], k[s]))) for s in range(L)]
            assert np.array_equal(S[i], np.array(exact, np.float64))


def test_scores_closed_form():
    """q_I[h] = e_h, w_h = h+1, k_s = e_(s mod 32)  =>  I[s] = (s mod 32) + 1."""
    L = 70
    q = np.zeros((1, 32, 128), np.float32)
    for h in range(32):
        q[0, h, h] = 1.0
    w = (np.arange(32, dtype=np.float32) + 1)[None, :]
    k = np.zeros((L, 128), np.float32)
    k[np.arange(L), np.arange(L) % 32] = 1.0
    S = oracle.indexer_scores(wl.bf16_from_f32(q), wl.bf16_from_f32(w), wl.bf16_from_f32(k),
                              np.zeros(1, np.int64), np.array([L], np.int32))
    assert np.array_equal(S[0], (np.arange(L) % 32 + 1).astype(np.float64))


def test_scores_causal_and_offset():
    """Entries past n_vis are untouched; rows read their own sequence via kv_start."""
    c = wl.make_case_numpy([50, 70], [(0, 10), (1, 70), (1, 33)], seed=3, n_plant=0)
    S = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=80)
    assert np.isnan(S[0, 10:]).all() and np.isnan(S[2, 33:]).all() and np.isnan(S[1, 70:]).all()
    # row 2 (seq 1, n_vis 33) equals row computed standalone on the slice of seq 1
    S2 = oracle.indexer_scores(c.q_I[2:3], c.w[2:3], c.k_I[50:], np.zeros(1, np.int64), np.array([33], np.int32))
    assert np.array_equal(S2[0], S[2, :33])


# ----------------------------------------------------------------------------- top-k

def brute_topk(score, n, k):
    order = sorted(range(n), key=lambda s: (-score[s], s))[:k]
    out = sorted(order) + [-1] * (k - min(k, n))
    return np.array(out, np.int32)


@pytest.mark.parametrize("k", [1, 3, 8])
def test_topk_bruteforce_with_ties(k):
    r = np.random.default_rng(k)
    for trial in range(200):
        n = int(r.integers(1, 65))
        score = r.integers(-3, 4, size=n).astype(np.float64)   # heavy ties
        got = oracle.topk(score[None, :], np.array([n], np.int32), k)[0]
        assert np.array_equal(got, brute_topk(score, n, k)), (trial, n)


def test_topk_all_equal_keeps_lowest_positions():
    for n, k in [(64, 8), (10, 3), (5, 8)]:
        got = oracle.topk(np.zeros((1, n)), np.array([n], np.int32), k)[0]
        expect = list(range(min(n, k))) + [-1] * max(0, k - n)
        assert got.tolist() == expect


def test_topk_signed_zero_is_a_tie():
    s = np.array([[-0.0, 0.0, -1.0]])
    assert oracle.topk(s, np.array([3], np.int32), 1)[0].tolist() == [0]
    s = np.array([[0.0, -0.0, -1.0]])
    assert oracle.topk(s, np.array([3], np.int32), 1)[0].tolist() == [0]


def test_topk_invariants_and_permutation():
    r = np.random.default_rng(9)
    n, k = 5000, 2048
    score = r.standard_normal(n)
    idx = oracle.topk(score[None], np.array([n], np.int32), k)[0]
    assert idx.size == k and (np.diff(idx) > 0).all() and idx.min() >= 0 and idx.max() < n
    sel = np.zeros(n, bool)
    sel[idx] = True
    assert score[sel].min() >= score[~sel].max()
    # distinct scores: the kept set does not depend on where positions are stored
    perm = r.permutation(n)
    idx_p = oracle.topk(score[perm][None], np.array([n], np.int32), k)[0]
    assert set(perm[idx_p].tolist()) == set(idx.tolist())


def test_topk_short_rows_pad():
    score = np.arange(10, dtype=np.float64)[None]
    got = oracle.topk(score, np.array([4], np.int32), 6)[0]
    assert got.tolist() == [0, 1, 2, 3, -1, -1]


def test_selected_count_matches_pages_dot_product_count():
    """Causal prefill keeps min(k, t+1) per query; at 1M context that is about
    1M x 2048 attention dot products against 10^12 dense (pages' figures)."""
    g = json.load(open(os.path.join(HERE, "golden", "pages_dot_product_counts.json")))
    N, k = 300, 64
    S = oracle.indexer_scores(*(lambda c: (c.q_I, c.w, c.k_I, c.kv_start, c.n_vis))(
        wl.make_case_numpy([N], [(0, t + 1) for t in range(N)], 11, n_plant=0)))
    idx = oracle.topk(S, np.arange(1, N + 1, dtype=np.int32), k)
    counts = (idx >= 0).sum(axis=1)
    assert counts.tolist() == [min(k, t + 1) for t in range(N)]
    n1m, k1m = g["context"], g["index_topk"]
    sparse = k1m * n1m - k1m * (k1m - 1) // 2          # sum_t min(k, t+1), t < n
    assert n1m * n1m == g["dense_dot_products_per_layer"]
    assert abs(sparse / (n1m * k1m) - 1) < 2e-3        # "1M x 2048"
    assert 450 < g["dense_dot_products_per_layer"] / sparse < 550   # "about 500x"


# ----------------------------------------------------------------------------- attention

def dense_reference(q, kv, n, scale):
    """Textbook softmax attention in latent form, written with scipy routines."""
    Q = f32(q).reshape(64, 576)
    K = f32(kv[:n])
    S = (Q @ K.T) * scale
    return softmax(S, axis=1) @ K[:, :512], logsumexp(S, axis=1)


def test_attention_equals_dense_when_topk_covers_context():
    r = np.random.default_rng(21)
    L = 90
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    q = wl.bf16_from_f32(r.standard_normal((3, 64, 576)).astype(np.float32))
    n_vis = np.array([1, 47, 90], np.int32)
    k = 128
    idx = np.full((3, k), -1, np.int32)
    for i, n in enumerate(n_vis):
        idx[i, :n] = np.arange(n)
    o, lse = oracle.sparse_mla(q, kv, np.zeros(3, np.int64), idx, 1 / 16)
    for i, n in enumerate(n_vis):
        ro, rl = dense_reference(q[i], kv, n, 1 / 16)
        assert np.max(np.abs(o[i] - ro)) < 1e-12
        assert np.max(np.abs(lse[i] - rl)) < 1e-12


def test_attention_rope_only_and_latent_only():
    r = np.random.default_rng(22)
    L = 40
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    qf = r.standard_normal((2, 64, 576)).astype(np.float32)
    qf[0, :, :512] = 0.0   # rope part alone decides
    qf[1, :, 512:] = 0.0   # latent part alone decides
    q = wl.bf16_from_f32(qf)
    idx = np.tile(np.arange(L, dtype=np.int32), (2, 1))
    o, lse = oracle.sparse_mla(q, kv, np.zeros(2, np.int64), idx, 1 / 16)
    for i in range(2):
        ro, rl = dense_reference(q[i], kv, L, 1 / 16)
        assert np.max(np.abs(o[i] - ro)) < 1e-12 and np.max(np.abs(lse[i] - rl)) < 1e-12


def test_attention_single_key_and_equal_scores():
    r = np.random.default_rng(23)
    L = 30
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    q = wl.bf16_from_f32(r.standard_normal((2, 64, 576)).astype(np.float32))
    idx = np.full((2, 8), -1, np.int32)
    idx[0, 3] = 17                       # one selected key -> o = c_kv[17]
    o, lse = oracle.sparse_mla(q, kv, np.zeros(2, np.int64), idx, 1 / 16)
    assert np.array_equal(o[0], np.tile(f32(kv[17, :512]), (64, 1)))
    s17 = (f32(q[0]) @ f32(kv[17])) / 16
    assert np.max(np.abs(lse[0] - s17)) < 1e-12
    # q = 0 -> all scores equal -> mean of the selected rows, lse = log(count)
    qz = np.zeros((1, 64, 576), np.uint16)
    sel = np.array([[2, 5, 11, 29, -1, -1]], np.int32)
    o, lse = oracle.sparse_mla(qz, kv, np.zeros(1, np.int64), sel, 1 / 16)
    mean = f32(kv[[2, 5, 11, 29], :512]).mean(axis=0)
    assert np.max(np.abs(o[0] - mean)) < 1e-12
    assert np.max(np.abs(lse[0] - np.log(4))) < 1e-12


def test_attention_weights_sum_to_one():
    """With every c_kv row equal to c, o = c * sum_j p_j, so o == c iff sum p = 1."""
    r = np.random.default_rng(24)
    L = 64
    kvf = r.standard_normal((L, 576)).astype(np.float32)
    c = r.standard_normal(512).astype(np.float32)
    kvf[:, :512] = c
    kv = wl.bf16_from_f32(kvf)
    q = wl.bf16_from_f32(r.standard_normal((1, 64, 576)).astype(np.float32) * 3)
    idx = np.arange(L, dtype=np.int32)[None]
    o, _ = oracle.sparse_mla(q, kv, np.zeros(1, np.int64), idx, 1 / 16)
    assert np.max(np.abs(o[0] - f32(kv[0, :512])[None])) < 1e-12


def test_attention_permutation_and_padding_invariance():
    r = np.random.default_rng(25)
    L = 200
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    q = wl.bf16_from_f32(r.standard_normal((1, 64, 576)).astype(np.float32))
    sel = np.sort(r.choice(L, 50, replace=False)).astype(np.int32)
    a = np.concatenate([sel, -np.ones(14, np.int32)])[None]
    b = np.concatenate([-np.ones(7, np.int32), r.permutation(sel), -np.ones(7, np.int32)])[None]
    oa, la = oracle.sparse_mla(q, kv, np.zeros(1, np.int64), a, 1 / 16)
    ob, lb = oracle.sparse_mla(q, kv, np.zeros(1, np.int64), b, 1 / 16)
    assert np.max(np.abs(oa - ob)) < 1e-12 and np.max(np.abs(la - lb)) < 1e-12


# ----------------------------------------------------------------------------- whole step

def test_forward_is_the_composition():
    c = small_case(seed=7, L=400, T=6, topk=64)
    o, lse, idx = oracle.forward_case(c, 1 / 16)
    S = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis)
    idx2 = oracle.topk(S, c.n_vis, c.topk)
    o2, lse2 = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx2, 1 / 16)
    assert np.array_equal(idx, idx2)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_forward_causal_future_keys_do_not_matter():
    c = small_case(seed=8, L=300, T=3, topk=32)
    o, lse, idx = oracle.forward_case(c, 1 / 16)
    nmax = int(c.n_vis.max())
    c.k_I[nmax:] = 0x3F80   # overwrite positions no row can see
    c.kv[nmax:] = 0x4000
    o2, lse2, idx2 = oracle.forward_case(c, 1 / 16)
    assert np.array_equal(idx, idx2) and np.array_equal(o, o2)


def test_forward_dense_when_topk_exceeds_context():
    c = small_case(seed=9, L=120, T=3, topk=256)
    o, lse, idx = oracle.forward_case(c, 1 / 16)
    for i in range(c.T):
        n = int(c.n_vis[i])
        assert idx[i, :n].tolist() == list(range(n)) and (idx[i, n:] == -1).all()
        ro, rl = dense_reference(c.q[i], c.kv, n, 1 / 16)
        assert np.max(np.abs(o[i] - ro)) < 1e-12 and np.max(np.abs(lse[i] - rl)) < 1e-12


def test_planted_positions_are_recalled():
    """Planted keys score ~2.3 against a noise maximum ~1.3, so every surviving
    plant must be kept (end-to-end invariant of the input recipe)."""
    c = wl.make_workload_numpy(0, scale=8)     # 4 queries over a 4096-row shared cache
    _, _, idx = oracle.forward_case(c, 1 / 16)
    for i in range(c.T):
        p = c.plants[i][c.plants[i] >= 0]
        assert p.size > 0
        assert np.isin(p, idx[i]).all()


# ---------------------------------------------------------------------------- dense + sparse branches
# ("GLM-5.2's DSA architecture: how dense and sparse attention split the work",
# section "DSA's core design": a sliding-window dense branch next to the sparse
# branch, fused per head by learned weights, here a caller-supplied gate.)

def _window_reference(qi, kv, ks, n, window, scale):
    """Dense attention of one row over its last `window` visible positions, with
    scipy's softmax / logsumexp (no oracle code)."""
    lo = max(0, n - window)
    K = f32(kv[ks + lo:ks + n])
    S = (f32(qi) @ K.T) * scale
    return softmax(S, axis=1) @ K[:, :512], logsumexp(S, axis=1)


def test_dense_sparse_gate_extremes_are_the_branches():
    r = np.random.default_rng(91)
    L = 700
    kv = wl.bf16_from_f32(r.standard_normal((L + 50, 576)).astype(np.float32))
    q = wl.bf16_from_f32(r.standard_normal((4, 64, 576)).astype(np.float32))
    kv_start = np.array([50, 50, 0, 10], np.int64)
    n_vis = np.array([700, 300, 5, 640], np.int32)
    idx = np.full((4, 96), -1, np.int32)
    for i, n in enumerate(n_vis):
        m = min(96, int(n))
        idx[i, :m] = np.sort(r.choice(int(n), m, replace=False))
    for window in (1, 64, 128, 1000):
        o1, ld, ls = oracle.dense_sparse(q, kv, kv_start, n_vis, idx, window, np.ones((4, 64)), 1 / 16)
        o0, ld0, ls0 = oracle.dense_sparse(q, kv, kv_start, n_vis, idx, window, np.zeros((4, 64)), 1 / 16)
        os_, lss = oracle.sparse_mla(q, kv, kv_start, idx, 1 / 16)
        assert np.array_equal(o0, os_) and np.array_equal(ls, lss)   # gate 0: the sparse branch alone
        for i, n in enumerate(n_vis):
            ro, rl = _window_reference(q[i], kv, int(kv_start[i]), int(n), window, 1 / 16)
            assert np.max(np.abs(o1[i] - ro)) < 1e-12                 # gate 1: the window alone
            assert np.max(np.abs(ld[i] - rl)) < 1e-12


def test_dense_sparse_gate_mixes_per_head():
    r = np.random.default_rng(92)
    L = 400
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    q = wl.bf16_from_f32(r.standard_normal((2, 64, 576)).astype(np.float32))
    kv_start = np.zeros(2, np.int64)
    n_vis = np.array([400, 250], np.int32)
    idx = np.stack([np.sort(r.choice(int(n), 64, replace=False)) for n in n_vis]).astype(np.int32)
    gate = r.uniform(0, 1, (2, 64))
    o, _, _ = oracle.dense_sparse(q, kv, kv_start, n_vis, idx, 32, gate, 1 / 16)
    os_, _ = oracle.sparse_mla(q, kv, kv_start, idx, 1 / 16)
    for i, n in enumerate(n_vis):
        ro, _ = _window_reference(q[i], kv, 0, int(n), 32, 1 / 16)
        for h in (0, 17, 63):
            want = gate[i, h] * ro[h] + (1 - gate[i, h]) * os_[i, h]
            assert np.max(np.abs(o[i, h] - want)) < 1e-12
    # a window covering the whole context is full dense attention
    o_full, _, _ = oracle.dense_sparse(q, kv, kv_start, n_vis, idx, 2048, np.ones((2, 64)), 1 / 16)
    for i, n in enumerate(n_vis):
        ro, _ = dense_reference(q[i], kv, int(n), 1 / 16)
        assert np.max(np.abs(o_full[i] - ro)) < 1e-12


# ------------------------------------------------------------------ block-level variant
# ("GLM-5: 744B parameters, 202K long context", section 2: 128-token blocks, a local
# branch over the query's block and its neighbours (O(N * 384)), an anchor block in
# every 16, the 16 most relevant blocks per query, fused with weights)

def _block_case(seed, n_vis, L=None, planted_block=None):
    r = np.random.default_rng(seed)
    n_vis = np.asarray(n_vis, np.int32)
    L = int(n_vis.max()) if L is None else L
    T = n_vis.shape[0]
    q_I = wl.bf16_from_f32((r.standard_normal((T, 32, 128)) / np.sqrt(128)).astype(np.float32))
    w = wl.bf16_from_f32(r.random((T, 32)).astype(np.float32))
    k_If = (r.standard_normal((L, 128)) / np.sqrt(128)).astype(np.float32)
    if planted_block is not None:
        # one key aligned with row 0's mean query direction: its block must be kept
        u = wl.bf16_to_f32(q_I[0]).mean(axis=0)
        k_If[planted_block * oracle.BLOCK + 5] = 3.0 * u / np.linalg.norm(u)
    k_I = wl.bf16_from_f32(k_If)
    q = wl.bf16_from_f32(r.standard_normal((T, 64, 576)).astype(np.float32))
    kv = wl.bf16_from_f32(r.standard_normal((L, 576)).astype(np.float32))
    return q_I, w, k_I, q, kv, np.zeros(T, np.int64), n_vis


def test_block_counts_match_the_pages_202k_figures():
    g = json.load(open(os.path.join(HERE, "golden", "pages_block_counts.json")))
    assert oracle.BLOCK == g["block_tokens"] and oracle.BLOCK_TOPK == g["dynamic_topk_blocks"]
    n = g["context_202k_blocks"] * g["block_tokens"]             # 202752 positions
    S = np.zeros((1, n))
    loc, anc, dyn, blk = oracle.block_branch_sets(S, np.array([n], np.int32))
    assert (n + oracle.BLOCK - 1) // oracle.BLOCK == g["context_202k_blocks"]
    assert np.count_nonzero(anc[0] >= 0) == g["context_202k_anchor_blocks"] * oracle.BLOCK
    assert loc.shape[1] == g["local_window_positions"]
    # equal scores everywhere: the lowest 16 blocks win the ties
    assert blk[0].tolist() == list(range(16))


def test_block_dynamic_branch_is_dense_when_16_blocks_cover_the_context():
    q_I, w, k_I, q, kv, ks, n_vis = _block_case(301, [1, 129, 2000, 16 * 128])
    g = np.zeros((4, 64, 3))
    g[:, :, 2] = 1.0
    o, lses, sets = oracle.block_sparse(q_I, w, k_I, q, kv, ks, n_vis, g, 1 / 16)
    for i, n in enumerate(n_vis):
        ro, rl = dense_reference(q[i], kv, int(n), 1 / 16)
        assert np.max(np.abs(o[i] - ro)) < 1e-12
        assert np.max(np.abs(lses[2][i] - rl)) < 1e-12


def test_block_local_branch_is_a_sliding_window():
    # the query's block up to itself plus the previous block: a window of
    # (t mod 128) + 1 + 128 positions (fewer at the start)
    q_I, w, k_I, q, kv, ks, n_vis = _block_case(302, [1, 100, 128, 129, 383, 1000, 4097])
    g = np.zeros((7, 64, 3))
    g[:, :, 0] = 1.0
    o, lses, _ = oracle.block_sparse(q_I, w, k_I, q, kv, ks, n_vis, g, 1 / 16)
    for i, n in enumerate(n_vis):
        t = int(n) - 1
        W = min(int(n), t % 128 + 1 + 128)
        ro, rl = _window_reference(q[i], kv, 0, int(n), W, 1 / 16)
        assert np.max(np.abs(o[i] - ro)) < 1e-12
        assert np.max(np.abs(lses[0][i] - rl)) < 1e-12


def test_block_anchor_branch_attends_the_first_block_of_every_16():
    q_I, w, k_I, q, kv, ks, n_vis = _block_case(303, [5000, 2049, 100])
    g = np.zeros((3, 64, 3))
    g[:, :, 1] = 1.0
    o, lses, sets = oracle.block_sparse(q_I, w, k_I, q, kv, ks, n_vis, g, 1 / 16)
    anc = sets[1]
    # t = 4999 is in block 39: anchors 0, 16, 32 -> 384 positions; t = 2048: anchors 0, 16
    # (block 16 holds only position 2048 so far); t = 99: block 0 up to 99
    assert np.count_nonzero(anc[0] >= 0) == 384 and np.count_nonzero(anc[1] >= 0) == 129
    assert np.count_nonzero(anc[2] >= 0) == 100
    K = f32(kv)
    for i, n in enumerate(n_vis):
        p = np.array([s for s in range(int(n)) if (s // 128) % 16 == 0])
        S = (f32(q[i]) @ K[p].T) / 16
        assert np.max(np.abs(o[i] - softmax(S, axis=1) @ K[p, :512])) < 1e-12
        assert np.max(np.abs(lses[1][i] - logsumexp(S, axis=1))) < 1e-12


def test_block_dynamic_selection_by_brute_force_and_planted_block():
    q_I, w, k_I, q, kv, ks, n_vis = _block_case(304, [6000, 6000, 3333], planted_block=41)
    S = oracle.indexer_scores(q_I, w, k_I, ks, n_vis)
    _, _, dyn, blk = oracle.block_branch_sets(S, n_vis)
    for i, n in enumerate(n_vis):
        n = int(n)
        nb = (n + 127) // 128
        best = [max(S[i, s] for s in range(b * 128, min(n, b * 128 + 128))) for b in range(nb)]
        want = sorted(sorted(range(nb), key=lambda b: (-best[b], b))[:16])
        assert blk[i].tolist() == want
        pos = [s for b in want for s in range(b * 128, min(n, b * 128 + 128))]
        assert dyn[i][:len(pos)].tolist() == pos and (dyn[i][len(pos):] == -1).all()
    assert 41 in blk[0].tolist()                                   # the planted key's block


def test_block_fusion_is_the_gated_sum_of_the_branches():
    q_I, w, k_I, q, kv, ks, n_vis = _block_case(305, [3000, 700])
    r = np.random.default_rng(306)
    g = r.uniform(0, 1, (2, 64, 3))
    o, _, sets = oracle.block_sparse(q_I, w, k_I, q, kv, ks, n_vis, g, 1 / 16)
    parts = [oracle.sparse_mla(q, kv, ks, idx, 1 / 16)[0] for idx in sets[:3]]
    for i in range(2):
        for h in (0, 31, 63):
            want = sum(g[i, h, b] * parts[b][i, h] for b in range(3))
            assert np.max(np.abs(o[i, h] - want)) < 1e-12
