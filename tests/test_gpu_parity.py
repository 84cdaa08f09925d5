"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Sizes span several 128-key tiles with ragged tails, every indexer schedule
(1, 4 and 8 queries per tile; split and wave sweeps), rows shorter and longer
than topk, ties, signed zeros, padded index lists and shared caches.
"""
import os
import zlib

import numpy as np
import pytest

import oracle
from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import workloads as wl

from gpu_util import (ATT_MAX_ABS, ATT_REL_L2, SCALE, SET_TOL_REL, assert_attention_close, assert_scores_close,
                      assert_selection_ok, gpu_attention, gpu_forward, gpu_scores, gpu_topk, reference_set, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _lib():
    from indexer_selected_sparse_dsa_b200 import build
    build.build()
    B.lib()


# ---------------------------------------------------------------------------- indexer

INDEXER_CASES = {
    # name: (seq_lens, queries)
    "one_row_ragged": ([700], [(0, 700)]),
    "shared_cache_4": ([1000], [(0, 1000), (0, 999), (0, 640), (0, 1)]),
    "mixed_sequences": ([300, 129, 1000], [(0, 300), (1, 129), (2, 1000), (2, 513), (0, 17), (2, 1000), (1, 1)]),
    "causal_prefill": ([600], [(0, t + 1) for t in range(600)]),
    "many_decode_rows": ([257] * 40, [(b, 257 - (b % 3)) for b in range(40)]),
}


@pytest.mark.parametrize("name", sorted(INDEXER_CASES))
@pytest.mark.parametrize("sweep", ["split", "wave"])
def test_indexer_scores_match_oracle(name, sweep, monkeypatch):
    monkeypatch.setenv("DSA_INDEXER_SWEEP", sweep)
    seq_lens, queries = INDEXER_CASES[name]
    c = wl.make_case_numpy(seq_lens, queries, seed=zlib.crc32(name.encode()) % 1000, n_plant=4)
    ld = (max(c.n_vis) + 3) // 4 * 4 + 4
    ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=ld)
    got = gpu_scores(to_dev(c), ld).cpu().numpy()
    assert_scores_close(got, ref, c.n_vis)
    for i, n in enumerate(c.n_vis):     # columns past n_vis are not written
        assert np.isnan(got[i, n:]).all(), f"row {i} wrote past n_vis"


@pytest.mark.parametrize("qmax", ["1", "4", "8"])
def test_indexer_every_tile_width(qmax, monkeypatch):
    monkeypatch.setenv("DSA_INDEXER_QMAX", qmax)
    c = wl.make_case_numpy([900, 400], [(0, 900), (0, 899), (0, 777), (1, 400), (1, 385), (0, 5)], seed=31, n_plant=4)
    ld = 904
    ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=ld)
    got = gpu_scores(to_dev(c), ld).cpu().numpy()
    assert_scores_close(got, ref, c.n_vis)


def test_indexer_bad_row_is_skipped_and_reported():
    import torch
    c = wl.make_case_numpy([300], [(0, 300), (0, 200)], seed=3, n_plant=0)
    d = to_dev(c)
    d["n_vis"][1] = 0            # invalid: a query always sees itself
    ld = 300
    scores = torch.full((2, ld), float("nan"), device="cuda")
    ws = B.workspace(B.DSA_OP_INDEXER, 2, ld, 0)
    B.dsa_indexer_scores(d["q_I"], d["w"], d["k_I"], d["kv_start"], d["n_vis"], scores, ws)
    with pytest.raises(B.DSAError) as e:
        B.dsa_sync_status()
    assert e.value.code == B.DSA_ERR_BAD_ROW
    s = scores.cpu().numpy()
    ref = oracle.indexer_scores(c.q_I[:1], c.w[:1], c.k_I, c.kv_start[:1], c.n_vis[:1], score_ld=ld)
    assert_scores_close(s[:1], ref, c.n_vis[:1])
    assert np.isnan(s[1]).all()
    B.dsa_sync_status()         # the status word was cleared


# ---------------------------------------------------------------------------- top-k

def _topk_case(kind, n, seed):
    r = np.random.default_rng(seed)
    if kind == "normal":
        return r.standard_normal(n).astype(np.float32)
    if kind == "ties":
        return r.integers(-4, 5, size=n).astype(np.float32)
    if kind == "equal":
        return np.full(n, 0.75, np.float32)
    if kind == "zeros":
        z = np.zeros(n, np.float32)
        z[r.random(n) < 0.5] = -0.0
        z[r.random(n) < 0.1] = 1.0
        return z
    if kind == "wide":
        return (r.standard_normal(n) * np.exp(r.uniform(-30, 30, n))).astype(np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["normal", "ties", "equal", "zeros", "wide"])
@pytest.mark.parametrize("k", [1, 7, 2048])
@pytest.mark.parametrize("split", [None, "4", "short"])
def test_topk_bit_exact(kind, k, split, monkeypatch):
    # split "4": every row over a cluster of 4 CTAs (a 20000-key row leaves one idle);
    # "short": the short-row kernel (256 threads per row, three rows per SM)
    if split == "short":
        monkeypatch.setenv("DSA_TOPK_KERNEL", "short")
    elif split:
        monkeypatch.setenv("DSA_TOPK_SPLIT", split)
    lens = [1, 5, k - 1 if k > 1 else 1, k, k + 1, 2047, 2049, 5000, 20000]
    ld = (max(lens) + 3) // 4 * 4
    S = np.full((len(lens), ld), np.nan, np.float32)
    for i, n in enumerate(lens):
        S[i, :n] = _topk_case(kind, n, seed=i * 7 + k)
    n_vis = np.array(lens, np.int32)
    ref = oracle.topk(S.astype(np.float64), n_vis, k)   # the same fp32 values, compared exactly
    got = gpu_topk(S, n_vis, k)
    for i in range(len(lens)):
        assert np.array_equal(got[i], ref[i]), f"{kind} k={k} row {i} n={lens[i]}"


@pytest.mark.parametrize("kind", ["normal", "ties", "equal", "zeros", "comb", "strided"])
@pytest.mark.parametrize("k", [7, 2048])
@pytest.mark.parametrize("split", [None, "2", "4", "short"])
def test_topk_dense_rows_exact(kind, k, split, monkeypatch):
    # rows from just above the on-chip candidate buffer (10240 keys) to 32769
    # keys, streamed by one CTA or a cluster (sampled threshold, cuts, merge);
    # "short": up to 32768 keys through the short-row kernel, whose buffer
    # (6144) the combs, equal rows and strided rows overflow or starve
    if split == "short":
        monkeypatch.setenv("DSA_TOPK_KERNEL", "short")
    elif split:
        monkeypatch.setenv("DSA_TOPK_SPLIT", split)
    lens = [10241, 16383, 30001, 32767, 32768] + ([] if split == "short" else [32769])
    ld = 32768 if split == "short" else 32772
    S = np.full((len(lens), ld), np.nan, np.float32)
    for i, n in enumerate(lens):
        if kind == "comb":      # a tie class straddling the k-th place, spread over the row
            S[i, :n] = np.where(np.arange(n) % 5 == 0, 1.0, np.arange(n) * -1e-6).astype(np.float32)
        elif kind == "strided":  # high scores exactly on a strided sample's positions: the sample
            st = max(1, n // 4096)  # threshold then admits fewer than k keys (the full radix select runs)
            r = np.random.default_rng(7 * i)
            S[i, :n] = np.where(np.arange(n) % st == 0, 1.0 + r.random(n), np.arange(n) * -1e-6).astype(np.float32)
        else:
            S[i, :n] = _topk_case(kind, n, seed=31 * i + k)
    n_vis = np.array(lens, np.int32)
    ref = oracle.topk(S.astype(np.float64), n_vis, k)
    got = gpu_topk(S, n_vis, k)
    for i in range(len(lens)):
        assert np.array_equal(got[i], ref[i]), f"{kind} k={k} row {i} n={lens[i]}"


def test_topk_short_row_batch_exact():
    # a prefill-like batch: enough rows (>= 2 x the SM count) of at most 32768
    # scores that the launcher picks the short-row kernel by itself; lengths
    # from 1 to 32768, every score kind, ties at the k-th place
    r = np.random.default_rng(77)
    T, ld, k = 320, 32768, 2048
    lens = np.concatenate([[1, 2, 2047, 2048, 2049, 6143, 6144, 6145, 32768],
                           r.integers(1, ld + 1, T - 9)]).astype(np.int32)
    kinds = ["normal", "ties", "equal", "zeros", "wide"]
    S = np.full((T, ld), np.nan, np.float32)
    for i, n in enumerate(lens):
        S[i, :n] = _topk_case(kinds[i % len(kinds)], int(n), seed=1000 + i)
    ref = oracle.topk(S.astype(np.float64), lens, k)
    got = gpu_topk(S, lens, k)
    for i in range(T):
        assert np.array_equal(got[i], ref[i]), f"row {i} n={lens[i]} kind={kinds[i % len(kinds)]}"


@pytest.mark.parametrize("path,split", [("filtered", "1"), ("filtered", "2"), ("filtered", "4"), ("full", "1"),
                                        ("full", "2")])
def test_topk_long_rows_exact(path, split, monkeypatch):
    monkeypatch.setenv("DSA_TOPK_SPLIT", split)
    if path == "full":
        monkeypatch.setenv("DSA_TOPK_KERNEL", "row")
    lens = [131072, 204800, 65537]
    ld = 204800
    S = np.full((3, ld), np.nan, np.float32)
    for i, n in enumerate(lens):
        S[i, :n] = _topk_case("normal" if i != 2 else "ties", n, 5 + i)
    n_vis = np.array(lens, np.int32)
    ref = oracle.topk(S.astype(np.float64), n_vis, 2048)
    assert np.array_equal(gpu_topk(S, n_vis, 2048), ref)


@pytest.mark.parametrize("split", ["1", "4"])
def test_topk_filter_fallbacks(split, monkeypatch):
    monkeypatch.setenv("DSA_TOPK_SPLIT", split)
    # rows where the sample threshold admits too many keys (all equal, sorted
    # ascending with a constant tail) or where the sample misses the top keys
    n, k = 50000, 2048
    S = np.zeros((4, n), np.float32)
    S[0] = 1.0                                           # every key equal
    S[1] = np.arange(n, dtype=np.float32)                # increasing: top keys at the end
    S[2, :] = 0.5
    S[2, 7::12] = 2.0                                    # a regular comb between sample points
    r = np.random.default_rng(3)
    S[3] = r.standard_normal(n).astype(np.float32)
    S[3, r.choice(n, 3000, replace=False)] = 9.0         # 3000 ties above everything else
    n_vis = np.full(4, n, np.int32)
    ref = oracle.topk(S.astype(np.float64), n_vis, k)
    assert np.array_equal(gpu_topk(S, n_vis, k), ref)


@pytest.mark.parametrize("k", [7, 2048])
@pytest.mark.parametrize("split", ["1", "2", "4"])
def test_topk_buffer_cuts_exact(k, split, monkeypatch):
    monkeypatch.setenv("DSA_TOPK_SPLIT", split)
    # rows whose candidates overflow the on-chip buffer while streaming, so it
    # is cut to its exact top-k (ties to lower positions) one or more times
    n = 300000
    r = np.random.default_rng(11 + k)
    rows = [
        np.arange(n, dtype=np.float32),                                   # every chunk beats the last
        np.full(n, 2.5, np.float32),                                      # one tie class
        (np.arange(n) // 1000).astype(np.float32),                        # ascending plateaus of ties
        (np.arange(n) * 1e-4 + r.standard_normal(n)).astype(np.float32),  # drift plus noise
        np.where(np.arange(n) % 3 == 0, 1.0, 0.0).astype(np.float32),     # comb of ties
        r.integers(0, 3, n).astype(np.float32),                           # three tie classes
    ]
    S = np.stack(rows)
    n_vis = np.full(len(rows), n, np.int32)
    n_vis[4] = n - 5                                                      # ragged tail
    ref = oracle.topk(S.astype(np.float64), n_vis, k)
    got = gpu_topk(S, n_vis, k)
    for i in range(len(rows)):
        assert np.array_equal(got[i], ref[i]), f"row {i}"


@pytest.mark.parametrize("kind", ["normal", "ties", "equal", "zeros", "wide"])
def test_topk_full_radix_path_bit_exact(kind, monkeypatch):
    monkeypatch.setenv("DSA_TOPK_KERNEL", "row")
    lens = [1, 2047, 2048, 2049, 5000, 20000]
    S = np.full((len(lens), 20000), np.nan, np.float32)
    for i, n in enumerate(lens):
        S[i, :n] = _topk_case(kind, n, seed=100 + i)
    n_vis = np.array(lens, np.int32)
    ref = oracle.topk(S.astype(np.float64), n_vis, 2048)
    assert np.array_equal(gpu_topk(S, n_vis, 2048), ref)


# ---------------------------------------------------------------------------- attention

def _attention_case(seed, L=3000, T=5, k=2048, pad=(0, 100, 1900, 2047, 0)):
    c = wl.make_case_numpy([L], [(0, L)] * T, seed=seed, n_plant=0)
    r = np.random.default_rng(seed)
    idx = np.full((T, k), -1, np.int32)
    for i in range(T):
        m = k - pad[i % len(pad)]
        idx[i, :m] = np.sort(r.choice(L, m, replace=False))
    return c, idx


@pytest.mark.parametrize("split", [False, True])
def test_attention_matches_oracle_on_given_indices(split):
    c, idx = _attention_case(41)
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx, split=split)
    assert_attention_close(o, lse, o_ref, lse_ref)


def test_attention_split_with_empty_tiles_and_large_logits():
    # splits whose tiles hold no valid index, and logits large enough that the
    # splits' running maxima differ by far more than the lazy-rescale margin
    c = wl.make_case_numpy([3000], [(0, 3000)] * 3, seed=46, n_plant=0)
    c.q = wl.bf16_from_f32(wl.bf16_to_f32(c.q) * 6.0)
    r = np.random.default_rng(46)
    idx = np.full((3, 2048), -1, np.int32)
    idx[0, :130] = np.sort(r.choice(3000, 130, replace=False))          # only the first tiles
    idx[1, 1900:] = np.sort(r.choice(3000, 148, replace=False))         # only the last tile
    idx[2] = np.sort(r.choice(3000, 2048, replace=False))
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx, split=True)
    assert_attention_close(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("split", [False, True])
def test_attention_ragged_topk_and_gaps(split):
    # topk not a multiple of 128, -1 holes inside the list, unsorted entries
    c = wl.make_case_numpy([800], [(0, 800)] * 3, seed=43, n_plant=0)
    r = np.random.default_rng(43)
    k = 300
    idx = r.choice(800, size=(3, k)).astype(np.int32)
    idx[0, ::7] = -1
    idx[1, :] = -1
    idx[1, 5] = 123                     # single key: o = c_kv[123]
    idx[2, 150:] = -1
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx, split=split)
    assert_attention_close(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("split", [False, True])
def test_attention_empty_row_and_large_logits(split):
    c = wl.make_case_numpy([500], [(0, 500)] * 2, seed=44, n_plant=0)
    qf = wl.bf16_to_f32(c.q) * 8.0     # logits up to ~ +-40: exercises the lazy rescale
    c.q = wl.bf16_from_f32(qf)
    idx = np.full((2, 512), -1, np.int32)
    idx[0] = np.arange(500, dtype=np.int32).tolist() + [-1] * 12
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx, split=split)
    assert_attention_close(o, lse, o_ref, lse_ref)
    assert (o[1] == 0).all() and np.isneginf(lse[1]).all()


def test_attention_more_rows_than_sms():
    """More rows than SMs (several waves of CTAs); ragged lists of 1 to 384 keys."""
    c = wl.make_case_numpy([1500], [(0, 1500)] * 300, seed=48, n_plant=0)
    r = np.random.default_rng(48)
    k = 384
    idx = np.full((300, k), -1, np.int32)
    for i in range(300):
        m = [384, 200, 1, 257][i % 4]
        idx[i, :m] = np.sort(r.choice(1500, m, replace=False))
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx, split=True)
    assert_attention_close(o, lse, o_ref, lse_ref)


def test_attention_per_row_cache_offsets():
    c = wl.make_case_numpy([700, 900, 300], [(0, 700), (1, 900), (2, 300), (1, 450)], seed=45, n_plant=0)
    r = np.random.default_rng(45)
    k = 640
    idx = np.full((4, k), -1, np.int32)
    for i, n in enumerate(c.n_vis):
        m = min(k, int(n))
        idx[i, :m] = np.sort(r.choice(int(n), m, replace=False))
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    o, lse = gpu_attention(to_dev(c), idx)
    assert_attention_close(o, lse, o_ref, lse_ref)


# ---------------------------------------------------------------------------- whole step

def _forward_check(c, k=2048):
    d = to_dev(c)
    maxn = int(max(c.n_vis))
    o, lse, idx = gpu_forward(d, maxn, k)
    S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=maxn)
    assert_selection_ok(idx, S_ref, c.n_vis, k)
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)   # on the GPU's index set
    assert_attention_close(o, lse, o_ref, lse_ref)
    for i in range(c.T):                          # planted positions are recalled
        p = c.plants[i][c.plants[i] >= 0]
        assert np.isin(p, idx[i]).all(), f"row {i}: planted position dropped"
    return idx


def test_forward_decode_shared_cache_scaled():
    _forward_check(wl.make_workload_numpy(0, scale=4))       # 4 queries over 8192 shared rows


def test_forward_decode_per_sequence_scaled():
    c = wl.make_case_numpy([6000] * 6, [(b, 6000 - 7 * b) for b in range(6)], seed=1)
    _forward_check(c)


def test_forward_causal_prefill_short_rows():
    # rows t < topk keep every prior position; later rows select
    c = wl.make_case_numpy([2600], [(0, t + 1) for t in range(0, 2600, 37)] + [(0, 2048), (0, 2049), (0, 2600)],
                           seed=2)
    idx = _forward_check(c)
    for i, n in enumerate(c.n_vis):
        if n <= 2048:
            assert idx[i, :n].tolist() == list(range(n))


def test_indexer_only_ranks():
    """The indexer's scores decide which positions attend, never how much: doubling
    w (exact in bf16) doubles every score exactly, and the selection, the output
    and the lse stay the same bit for bit ("2026 LLM architecture overview (2):
    DSA and MoE of GLM 5 / DSV3.2", section 2.2)."""
    import torch
    c = wl.make_case_numpy([6000] * 3, [(b, 6000 - 5 * b) for b in range(3)], seed=91)
    d = to_dev(c)
    o1, lse1, idx1 = gpu_forward(d, 6000, 2048)
    d2 = dict(d)
    d2["w"] = (d["w"].float() * 2).to(torch.bfloat16)
    assert torch.equal(d2["w"].float(), d["w"].float() * 2)
    o2, lse2, idx2 = gpu_forward(d2, 6000, 2048)
    assert np.array_equal(idx1, idx2)
    assert np.array_equal(o1, o2) and np.array_equal(lse1, lse2)


def test_forward_ragged_decode_scaled():
    _forward_check(wl.make_workload_numpy(3, scale=32))


# ---------------------------------------------------------------------------- IndexShare

@pytest.mark.parametrize("split", [False, True])
def test_indexshare_shared_layers_match_oracle(split):
    """A group of four layers (N^2, section "IndexShare"): the full layer runs the
    whole step; three further layers attend over its index set with their own
    queries and latent caches and must match the oracle's attention on that set."""
    import torch
    c = wl.make_case_numpy([6000], [(0, 6000), (0, 5000), (0, 2100), (0, 900), (0, 1)], seed=71)
    d = to_dev(c)
    o0, lse0, idx = gpu_forward(d, 6000, 2048)
    o0_ref, lse0_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, wl.SCALE)
    assert_attention_close(o0, lse0, o0_ref, lse0_ref)
    for layer in (1, 2, 3):
        q_l, kv_l = wl.make_shared_layer_numpy(c, layer)
        dl = dict(d)
        dl["q"] = torch.from_numpy(q_l.view(np.int16)).view(torch.bfloat16).cuda()
        dl["kv"] = torch.from_numpy(kv_l.view(np.int16)).view(torch.bfloat16).cuda()
        o, lse = gpu_attention(dl, idx, split=split)
        o_ref, lse_ref = oracle.sparse_mla(q_l, kv_l, c.kv_start, idx, wl.SCALE)
        assert_attention_close(o, lse, o_ref, lse_ref)
        assert not np.allclose(o, o0)   # the layers differ; only the index set is shared


# ---------------------------------------------------------------------------- dense + sparse branches

@pytest.mark.parametrize("window", [1, 128, 700, 2048])
def test_dense_sparse_matches_oracle(window):
    """Two branches fused by a per-head gate ("GLM-5.2's DSA architecture: how dense
    and sparse attention split the work", section "DSA's core design")."""
    import torch
    c = wl.make_case_numpy([3000], [(0, 3000), (0, 2500), (0, 1000), (0, 130), (0, 1)], seed=93, n_plant=0)
    r = np.random.default_rng(94 + window)
    k = 2048
    idx = np.full((c.T, k), -1, np.int32)
    for i, n in enumerate(c.n_vis):
        m = min(k, int(n)) - (100 if n > 2100 else 0)
        idx[i, :m] = np.sort(r.choice(int(n), m, replace=False))
    gate = r.uniform(0, 1, (c.T, 64)).astype(np.float32)
    gate[1] = 0.0
    gate[2] = 1.0
    d = to_dev(c)
    o = torch.full((c.T, 64, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse_d = torch.full((c.T, 64), float("nan"), dtype=torch.float32, device="cuda")
    lse_s = torch.full((c.T, 64), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.workspace(B.DSA_OP_DENSE_SPARSE, c.T, 0, 0)
    B.dsa_dense_sparse_attn(d["q"], d["kv"], d["kv_start"], d["n_vis"], torch.from_numpy(idx).cuda(), window,
                            torch.from_numpy(gate).cuda(), SCALE, o, lse_d, lse_s, ws)
    B.dsa_sync_status()
    o_ref, ld_ref, ls_ref = oracle.dense_sparse(c.q, c.kv, c.kv_start, c.n_vis, idx, window, gate.astype(np.float64),
                                                SCALE)
    assert_attention_close(o.cpu().numpy(), lse_d.cpu().numpy(), o_ref, ld_ref)
    assert_attention_close(o.cpu().numpy(), lse_s.cpu().numpy(), o_ref, ls_ref)


# ---------------------------------------------------------------------------- streamed selection

STREAM_CASES = {
    # the query tile's candidate buffers shrink several times (rows much longer than 8192)
    "long_shared": lambda: wl.make_case_numpy([30000], [(0, 30000), (0, 29999), (0, 25000), (0, 9000), (0, 2048),
                                                        (0, 2049), (0, 100), (0, 1)], seed=61),
    "scaled_chunked_prefill": lambda: wl.make_workload_numpy(4, scale=64),
    "mixed_sequences": lambda: wl.make_case_numpy([20000, 5000, 12000], [(0, 20000), (1, 5000), (2, 12000),
                                                                          (2, 11000), (0, 19999)], seed=62),
}


@pytest.mark.parametrize("name", sorted(STREAM_CASES))
def test_forward_streamed_selection_equals_materialized(name, monkeypatch):
    c = STREAM_CASES[name]()
    d = to_dev(c)
    maxn = int(max(c.n_vis))
    monkeypatch.setenv("DSA_FORWARD_MODE", "materialize")
    o_m, lse_m, idx_m = gpu_forward(d, maxn, 2048)
    monkeypatch.setenv("DSA_FORWARD_MODE", "stream")
    o_s, lse_s, idx_s = gpu_forward(d, maxn, 2048)
    assert np.array_equal(idx_m, idx_s)
    assert np.array_equal(o_m, o_s) and np.array_equal(lse_m, lse_s)
    S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=maxn)
    assert_selection_ok(idx_s, S_ref, c.n_vis, 2048)
    for i in range(c.T):
        p = c.plants[i][c.plants[i] >= 0]
        assert np.isin(p, idx_s[i]).all()


def test_forward_streamed_ties_go_to_lowest_positions(monkeypatch):
    # keys of the second sequence are all zero: every score is exactly 0, so the
    # selection must be positions 0..2047 in both modes
    c = wl.make_case_numpy([12000, 15000], [(0, 12000), (1, 15000), (1, 9000)], seed=63, n_plant=0)
    c.k_I[12000:] = 0
    d = to_dev(c)
    monkeypatch.setenv("DSA_FORWARD_MODE", "stream")
    _, _, idx = gpu_forward(d, 15000, 2048)
    assert idx[1].tolist() == list(range(2048)) and idx[2].tolist() == list(range(2048))
    monkeypatch.setenv("DSA_FORWARD_MODE", "materialize")
    _, _, idx_m = gpu_forward(d, 15000, 2048)
    assert np.array_equal(idx, idx_m)


def _seeded_all_equal():
    c = wl.make_case_numpy([140000], [(0, 140000), (0, 139000), (0, 131072), (0, 20000)], seed=66, n_plant=0)
    c.k_I[:] = c.k_I[0]          # every score of a query is the same value
    return c


# One query tile over more than 128K keys: its filters are seeded from 64 sampled key units.
SEEDED_CASES = {
    "seeded_long": lambda: wl.make_case_numpy(
        [200000], [(0, 200000), (0, 199999), (0, 180000), (0, 150000), (0, 131072), (0, 70000), (0, 9000),
                   (0, 3000)], seed=64),
    "seeded_two_tiles": lambda: wl.make_case_numpy(
        [160000], [(0, 160000 - 3 * i) for i in range(11)], seed=65),
    "seeded_all_equal": _seeded_all_equal,
}


@pytest.mark.parametrize("mode", ["1", "2", "0"])
@pytest.mark.parametrize("name", sorted(SEEDED_CASES))
def test_indexer_topk_seeded_equals_scores_then_topk(name, mode, monkeypatch):
    """Seeded filters (mode 1), seeds at the sample maximum that send rows to the
    redo sweep (mode 2), and no seeding (mode 0) all select exactly what
    dsa_indexer_scores + dsa_topk select."""
    monkeypatch.setenv("DSA_STREAM_SAMPLE", mode)
    _check_indexer_topk(SEEDED_CASES[name]())


@pytest.mark.parametrize("name", sorted(STREAM_CASES))
def test_indexer_topk_equals_scores_then_topk(name):
    """The fused entry point selects exactly what dsa_indexer_scores + dsa_topk select."""
    _check_indexer_topk(STREAM_CASES[name]())


def _check_indexer_topk(c):
    import torch
    d = to_dev(c)
    T, maxn, k = c.T, int(max(c.n_vis)), 2048
    ld = (maxn + 3) // 4 * 4
    scores = torch.empty((T, ld), dtype=torch.float32, device="cuda")
    B.dsa_indexer_scores(d["q_I"], d["w"], d["k_I"], d["kv_start"], d["n_vis"], scores,
                         B.workspace(B.DSA_OP_INDEXER, T, ld, 0))
    idx_a = torch.empty((T, k), dtype=torch.int32, device="cuda")
    B.dsa_topk(scores, d["n_vis"], k, idx_a)
    idx_b = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    B.dsa_indexer_topk(d["q_I"], d["w"], d["k_I"], d["kv_start"], d["n_vis"], maxn, k, idx_b,
                       B.workspace(B.DSA_OP_INDEXER_TOPK, T, maxn, k))
    B.dsa_sync_status()
    assert np.array_equal(idx_a.cpu().numpy(), idx_b.cpu().numpy())


# ------------------------------------------------------------------ block-level variant

@pytest.mark.parametrize("seed", [61, 62])
def test_block_sparse_matches_oracle(seed):
    """dsa_block_sparse_attn: the dynamic blocks equal the oracle's selection on the
    GPU's own fp32 scores (the float decision taken in one precision) and differ
    from the fp64 oracle's only inside the tie band; the fused output and each
    branch's lse match the oracle run on the GPU's blocks."""
    import torch
    lens = [20000, 7000]
    queries = [(0, 1), (0, 100), (0, 129), (0, 2049), (0, 5000), (0, 20000), (1, 7000), (1, 3000)]
    c = wl.make_case_numpy(lens, queries, seed=seed, n_plant=16)
    d = to_dev(c)
    T = c.T
    max_n = int(c.n_vis.max())
    r = np.random.default_rng(seed)
    gates = r.uniform(0, 1, (T, 64, 3)).astype(np.float32)
    o = torch.full((T, 64, 512), float("nan"), device="cuda")
    lse = torch.full((3, T, 64), float("nan"), device="cuda")
    blocks = torch.full((T, B.BLOCK_TOPK), -7, dtype=torch.int32, device="cuda")
    ws = B.workspace(B.DSA_OP_BLOCK_SPARSE, T, max_n, 0)
    B.dsa_block_sparse_attn(d["q_I"], d["w"], d["k_I"], d["q"], d["kv"], d["kv_start"], d["n_vis"], max_n,
                            torch.from_numpy(gates).cuda(), SCALE, o, lse, blocks, ws)
    B.dsa_sync_status()
    ld = (max_n + 3) // 4 * 4
    off = B.dsa_workspace_size(B.DSA_OP_INDEXER, T, max_n, 0)
    S_gpu = ws[off:off + T * ld * 4].view(torch.float32).view(T, ld).cpu().numpy().astype(np.float64)
    sets = oracle.block_branch_sets(S_gpu, c.n_vis)
    g_blocks = blocks.cpu().numpy()
    np.testing.assert_array_equal(g_blocks, sets[3])
    # against the fp64 oracle: only swaps of blocks whose scores tie within the band
    S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis)
    assert_scores_close(S_gpu[:, :max_n], S_ref, c.n_vis)
    bs = oracle.block_scores(S_ref, c.n_vis)
    _, _, _, ref_blocks = oracle.block_branch_sets(S_ref, c.n_vis)
    for i in range(T):
        diff = set(ref_blocks[i][ref_blocks[i] >= 0].tolist()) ^ set(g_blocks[i][g_blocks[i] >= 0].tolist())
        if diff:
            kth = np.sort(bs[i])[::-1][15]
            band = SET_TOL_REL * np.max(np.abs(S_ref[i, :c.n_vis[i]]))
            assert all(abs(bs[i][b] - kth) <= band for b in diff), f"row {i}: blocks {diff}"
    # attention: the oracle on the GPU's branch sets, fused with the same gates
    outs, lses = [], []
    for idx in sets[:3]:
        ob, lb = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
        outs.append(ob)
        lses.append(lb)
    o_ref = sum(gates.astype(np.float64)[:, :, b, None] * outs[b] for b in range(3))
    g_lse = lse.cpu().numpy()
    o_np = o.cpu().numpy()
    for i in range(T):
        dlt = o_np[i].astype(np.float64) - o_ref[i]
        assert np.max(np.abs(dlt)) <= ATT_MAX_ABS, f"row {i}"
        assert np.linalg.norm(dlt) <= ATT_REL_L2 * max(np.linalg.norm(o_ref[i]), 1e-30), f"row {i}"
        for b in range(3):
            fin = np.isfinite(lses[b][i])
            assert np.array_equal(fin, np.isfinite(g_lse[b][i])), f"row {i} branch {b}: lse finiteness"
            assert np.max(np.abs(g_lse[b][i][fin] - lses[b][i][fin])) <= ATT_MAX_ABS, f"row {i} branch {b}: lse"
    # every surviving planted position's block is kept by its row's dynamic branch
    for i in range(T):
        p = c.plants[i][c.plants[i] >= 0]
        assert np.isin(p // 128, g_blocks[i]).all(), f"row {i}: a planted block was dropped"


# ---------------------------------------------------------------------------- fused decode step

def _fused_case(name):
    if name == "shared_cache_scaled":
        return wl.make_workload_numpy(0, scale=4)
    if name == "mixed_tiles":
        # rows 0-3 share a sequence (one query tile), row 4 the same sequence (next tile),
        # then one row per sequence; rows shorter and longer than topk
        return wl.make_case_numpy([6000, 2048, 100, 3000],
                                  [(0, 6000), (0, 5999), (0, 4000), (0, 2049), (0, 1), (1, 2048), (2, 100),
                                   (3, 3000)], seed=71)
    if name == "all_ties":
        # every key of the second sequence is zero: its scores tie at 0 and the
        # lowest positions win; the first sequence's keys take 5 values
        c = wl.make_case_numpy([9000, 15000], [(0, 9000), (1, 15000), (1, 9000)], seed=72, n_plant=0)
        c.k_I[9000:] = 0
        c.k_I[:9000] = c.k_I[np.arange(9000) % 5]
        return c
    if name == "short_rows":
        return wl.make_case_numpy([2048], [(0, 1), (0, 128), (0, 129), (0, 2048)], seed=73)
    if name == "long_rows":  # the longest context the one-launch step takes
        return wl.make_case_numpy([32768], [(0, 32768), (0, 30001)], seed=74)
    if name == "eight_sequences":  # the largest batch: 8 query tiles of one row, 128 attention tiles
        return wl.make_case_numpy([32768] * 8, [(b, 32768 - 1000 * b) for b in range(8)], seed=76)
    raise KeyError(name)


FUSED_CASES = ["shared_cache_scaled", "mixed_tiles", "all_ties", "short_rows", "long_rows", "eight_sequences"]


@pytest.fixture
def fused_on(monkeypatch):
    monkeypatch.setenv("DSA_DECODE_FUSED", "1")


@pytest.mark.parametrize("name", FUSED_CASES)
def test_fused_decode_matches_oracle(name, fused_on):
    """With DSA_DECODE_FUSED=1, dsa_forward on batches of at most 8 rows runs the one-launch decode step.
    Its selection is checked bit-exactly against the oracle's top-k on the
    kernel's own fp32 scores (read back from the workspace) and against fp64
    scores within the tie band; the attention against the oracle on the
    kernel's index set."""
    import torch
    c = _fused_case(name)
    d = to_dev(c)
    T, k = c.T, 2048
    maxn = int(max(c.n_vis))
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((T, 64), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws = B.workspace(B.DSA_OP_FORWARD, T, maxn, k)
    B.dsa_forward(d["q_I"], d["w"], d["k_I"], d["q"], d["kv"], d["kv_start"], d["n_vis"], maxn, k, SCALE,
                  o, lse, idx, ws)
    B.dsa_sync_status()
    ld = (maxn + 3) // 4 * 4
    off = B.dsa_workspace_size(B.DSA_OP_INDEXER, T, maxn, k) // 4
    S_gpu = ws.view(torch.float32)[off:off + T * ld].view(T, ld).cpu().numpy()
    idx, o, lse = idx.cpu().numpy(), o.cpu().numpy(), lse.cpu().numpy()
    S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=ld)
    assert_scores_close(S_gpu, S_ref, c.n_vis)
    S_own = np.where(np.arange(ld)[None, :] < c.n_vis[:, None], S_gpu, 0).astype(np.float64)
    assert np.array_equal(idx, oracle.topk(S_own, c.n_vis, k)), "selection differs on the kernel's own scores"
    assert_selection_ok(idx, S_ref, c.n_vis, k)
    o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, SCALE)
    assert_attention_close(o, lse, o_ref, lse_ref)
    for i in range(T):
        p = c.plants[i][c.plants[i] >= 0]
        assert np.isin(p, idx[i]).all(), f"row {i}: planted position dropped"
    if name == "all_ties":
        assert idx[1].tolist() == list(range(2048)) and idx[2].tolist() == list(range(2048))


def test_fused_decode_skips_a_bad_row(fused_on):
    import torch
    c = wl.make_case_numpy([3000], [(0, 3000), (0, 2500), (0, 100)], seed=75)
    d = to_dev(c)
    d["n_vis"][1] = 5000                      # beyond the declared max_n_vis and the cache
    T, k, maxn = 3, 2048, 3000
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((T, 64), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws = B.workspace(B.DSA_OP_FORWARD, T, maxn, k)
    B.dsa_forward(d["q_I"], d["w"], d["k_I"], d["q"], d["kv"], d["kv_start"], d["n_vis"], maxn, k, SCALE,
                  o, lse, idx, ws)
    with pytest.raises(B.DSAError) as e:
        B.dsa_sync_status()
    assert e.value.code == B.DSA_ERR_BAD_ROW
    idx, o, lse = idx.cpu().numpy(), o.cpu().numpy(), lse.cpu().numpy()
    assert (idx[1] == -1).all() and (o[1] == 0).all() and np.isneginf(lse[1]).all()
    good = [0, 2]
    n_good = c.n_vis[good]
    S_ref = oracle.indexer_scores(c.q_I[good], c.w[good], c.k_I, c.kv_start[good], n_good, score_ld=maxn)
    assert_selection_ok(idx[good], S_ref, n_good, k)
    o_ref, lse_ref = oracle.sparse_mla(c.q[good], c.kv, c.kv_start[good], idx[good], SCALE)
    assert_attention_close(o[good], lse[good], o_ref, lse_ref)


@pytest.mark.parametrize("name", ["mixed_tiles", "long_rows"])
def test_fused_and_separate_kernels_agree(name, monkeypatch):
    """The one-launch step and the separate kernels select the same sets up to
    near-ties (their fp32 head sums differ in order) and give the same attention."""
    c = _fused_case(name)
    d = to_dev(c)
    maxn = int(max(c.n_vis))
    monkeypatch.setenv("DSA_DECODE_FUSED", "1")
    o_f, lse_f, idx_f = gpu_forward(d, maxn, 2048)
    monkeypatch.setenv("DSA_DECODE_FUSED", "0")
    o_s, lse_s, idx_s = gpu_forward(d, maxn, 2048)
    S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, score_ld=maxn)
    for i, n in enumerate(c.n_vis):
        K = min(2048, int(n))
        diff = np.setxor1d(idx_f[i, :K], idx_s[i, :K])
        if diff.size:
            _, kth = reference_set(S_ref[i, :n], K)
            assert (np.abs(S_ref[i, diff] - kth) <= SET_TOL_REL * np.max(np.abs(S_ref[i, :n]))).all()
        else:
            assert np.max(np.abs(o_f[i] - o_s[i])) <= ATT_MAX_ABS
