"""Helpers shared by the GPU tests: move seeded cases to the device and
compare the CUDA path with the oracle under the stated tolerances."""
import numpy as np

from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import workloads as wl

SCALE = wl.SCALE
IDX_TOL_REL = 2e-2        # indexer: |dI| <= 2e-2 * max|I|
SET_TOL_REL = 1e-3        # selection may differ only within 1e-3 * max|I| of the k-th score
ATT_MAX_ABS = 2e-2        # attention: max-abs
ATT_REL_L2 = 5e-3         # attention: relative L2


def to_dev(c):
    import torch

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    return dict(q_I=bf(c.q_I), w=bf(c.w), k_I=bf(c.k_I), q=bf(c.q), kv=bf(c.kv),
                kv_start=torch.from_numpy(np.asarray(c.kv_start, np.int64)).cuda(),
                n_vis=torch.from_numpy(np.asarray(c.n_vis, np.int32)).cuda())


def gpu_scores(d, score_ld, fill=float("nan")):
    import torch
    T = d["n_vis"].shape[0]
    scores = torch.full((T, score_ld), fill, dtype=torch.float32, device="cuda")
    ws = B.workspace(B.DSA_OP_INDEXER, T, score_ld, 0)
    B.dsa_indexer_scores(d["q_I"], d["w"], d["k_I"], d["kv_start"], d["n_vis"], scores, ws)
    B.dsa_sync_status()
    return scores


def gpu_topk(scores_np_f32, n_vis, k):
    import torch
    s = torch.from_numpy(np.ascontiguousarray(scores_np_f32, np.float32)).cuda()
    nv = torch.from_numpy(np.asarray(n_vis, np.int32)).cuda()
    idx = torch.empty((s.shape[0], k), dtype=torch.int32, device="cuda")
    B.dsa_topk(s, nv, k, idx)
    B.dsa_sync_status()
    return idx.cpu().numpy()


def gpu_attention(d, idx_np, scale=SCALE, split=False):
    """split=True passes the workspace, so rows may be spread over several CTAs."""
    import torch
    T, k = idx_np.shape
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, np.int32)).cuda()
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((T, 64), float("nan"), dtype=torch.float32, device="cuda")
    ws = B.workspace(B.DSA_OP_SPARSE_MLA, T, 0, k) if split else None
    B.dsa_sparse_mla_attn(d["q"], d["kv"], d["kv_start"], idx, scale, o, lse, ws)
    B.dsa_sync_status()
    return o.cpu().numpy(), lse.cpu().numpy()


def gpu_forward(d, max_n_vis, k, scale=SCALE):
    import torch
    T = d["n_vis"].shape[0]
    o = torch.full((T, 64, 512), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((T, 64), float("nan"), dtype=torch.float32, device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    ws = B.workspace(B.DSA_OP_FORWARD, T, max_n_vis, k)
    B.dsa_forward(d["q_I"], d["w"], d["k_I"], d["q"], d["kv"], d["kv_start"], d["n_vis"], max_n_vis, k, scale,
                  o, lse, idx, ws)
    B.dsa_sync_status()
    return o.cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()


def assert_scores_close(got, ref, n_vis):
    for i, n in enumerate(n_vis):
        r = ref[i, :n]
        g = got[i, :n].astype(np.float64)
        tol = IDX_TOL_REL * np.max(np.abs(r))
        err = np.max(np.abs(g - r))
        assert np.isfinite(g).all(), f"row {i}: non-finite score"
        assert err <= tol, f"row {i}: max |dI| {err:.3e} > {tol:.3e}"


def assert_attention_close(o, lse, o_ref, lse_ref, rows=None):
    rows = range(o.shape[0]) if rows is None else rows
    for i in rows:
        d = o[i].astype(np.float64) - o_ref[i]
        mabs = np.max(np.abs(d))
        rel = np.linalg.norm(d) / max(np.linalg.norm(o_ref[i]), 1e-30)
        assert mabs <= ATT_MAX_ABS, f"row {i}: max-abs {mabs:.3e}"
        assert rel <= ATT_REL_L2, f"row {i}: rel-L2 {rel:.3e}"
        fin = np.isfinite(lse_ref[i])
        assert np.array_equal(fin, np.isfinite(lse[i])), f"row {i}: lse finiteness differs"
        if fin.any():
            assert np.max(np.abs(lse[i][fin] - lse_ref[i][fin])) <= ATT_MAX_ABS, f"row {i}: lse"


def reference_set(r, K):
    """The oracle's kept set of one row: the unique top-K positions of the order
    (score descending, position ascending), and the K-th score."""
    n = r.shape[0]
    if K >= n:
        return np.arange(n), (np.min(r) if n else 0.0)
    kth = np.partition(r, n - K)[n - K]          # K-th largest value
    above = np.nonzero(r > kth)[0]
    tied = np.nonzero(r == kth)[0]               # ascending positions: the lowest win
    return np.sort(np.concatenate([above, tied[:K - above.size]])), kth


def assert_selection_ok(idx_gpu, scores_ref, n_vis, k, rows=None):
    """The GPU's kept set may differ from the oracle's only at positions whose
    oracle score lies within 1e-3 * max|I| of the oracle's k-th score; and it
    must be a valid selection: ascending, -1 padded, size min(k, n_vis)."""
    for i, n in enumerate(n_vis):
        name = i if rows is None else rows[i]
        g = idx_gpu[i]
        K = min(k, int(n))
        assert (g[K:] == -1).all(), f"row {name}: padding"
        sel = g[:K]
        assert (sel >= 0).all() and (sel < n).all(), f"row {name}: out of range"
        assert (np.diff(sel) > 0).all(), f"row {name}: not strictly ascending"
        r = scores_ref[i, :n]
        ref, kth = reference_set(r, K)
        band = SET_TOL_REL * np.max(np.abs(r))
        diff = np.setxor1d(ref, sel)
        if diff.size:
            gap = np.abs(r[diff] - kth)
            assert (gap <= band).all(), \
                f"row {name}: position {int(diff[np.argmax(gap)])} differs with score gap {gap.max():.3e} > {band:.3e}"


def host_rows(c, rows, with_kv=True):
    """Compact host copies (uint16 bf16 bits) of some query rows of a torch case:
    their query tensors and only their own visible cache prefixes, re-based so
    row j's sequence starts at the returned kv_start[j].  with_kv=False skips
    the latent cache (kv is then None): enough for the indexer side."""
    import torch

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    ks = c.kv_start.cpu().numpy()
    nv = c.n_vis.cpu().numpy()
    kI, kv, starts = [], [], []
    off = 0
    seen = {}   # rows of one sequence share one copy of its prefix
    for r in rows:
        s0 = int(ks[r])
        n = int(max(nv[q] for q in rows if int(ks[q]) == s0))
        if s0 not in seen:
            kI.append(u16(c.k_I[s0:s0 + n]))
            if with_kv:
                kv.append(u16(c.kv[s0:s0 + n]))
            seen[s0] = off
            off += n
        starts.append(seen[s0])
    return dict(q_I=u16(c.q_I[rows]), w=u16(c.w[rows]), q=u16(c.q[rows]), k_I=np.concatenate(kI),
                kv=np.concatenate(kv) if with_kv else None, kv_start=np.array(starts, np.int64), n_vis=nv[rows].astype(np.int32),
                plants=c.plants[rows])


def host_selected_rows(c, rows, idx_rows):
    """Host copies for checking the attention of some query rows: their queries
    and only the latent-cache rows their index lists select, laid out so that
    row j's selected rows start at kv_start[j] = j * k and its list becomes
    0, 1, 2, ... (-1 padding kept).  The GPU's lists are ascending and unique,
    so the oracle sees the same set in the same order."""
    import torch

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    idx_rows = np.asarray(idx_rows, np.int32)
    R, k = idx_rows.shape
    dev = c.kv.device
    ks = c.kv_start[torch.as_tensor(rows, dtype=torch.long, device=dev)]
    it = torch.from_numpy(idx_rows).to(dev).long()
    valid = it >= 0
    src = torch.where(valid, ks[:, None] + it, torch.zeros_like(it))
    kv_sel = c.kv[src.reshape(-1)].reshape(R * k, c.kv.shape[1])
    idx_local = np.where(idx_rows >= 0, np.arange(k, dtype=np.int32)[None, :], -1).astype(np.int32)
    return dict(q=u16(c.q[torch.as_tensor(rows, dtype=torch.long, device=dev)]), kv=u16(kv_sel),
                kv_start=(np.arange(R, dtype=np.int64) * k), idx=idx_local)
