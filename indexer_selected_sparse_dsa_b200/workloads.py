"""Seeded synthetic inputs for the DSA sparse-attention step.

This module only draws random numbers and lays them out; it contains none of
the method's arithmetic (no indexer score, no selection, no softmax).  Both
the CUDA path and the fp64 oracle consume the exact bf16 bit patterns it
produces, so the two sides share inputs and nothing else.

Shapes follow the GLM-5 / DeepSeek-V3.2 attention config table (page
"2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.1): 32 indexer heads of dim
128 (section 2.2), 64 MLA heads, kv_lora_rank 512, qk_rope_head_dim 64,
index_topk 2048.  The value laws are:

* q_I, k_I ~ N(0,1)/sqrt(128) per component; w ~ U(0,1);
* q = (q_lat || q_rope) and kv = (c_kv || k_rope) ~ N(0,1);
* planted keys: for query t, P positions of its causal prefix get
  k_I = 0.8 * unit(mean_h q_I[t,h]) + 0.2 * n,  n ~ N(0,1)/sqrt(128),
  written in ascending query order (a later query overwrites an earlier one
  on a shared cache; ``plants`` records only the survivors).

Two back ends draw from the same recipe: ``numpy`` (PCG64, exact across
machines; small and medium cases) and ``torch`` (a seeded device generator,
used for the multi-GB workloads).  They do not promise identical values to
each other; each is deterministic for a given seed.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

H_I = 32        # indexer heads
D_I = 128       # indexer head dim
H = 64          # MLA heads
D_C = 512       # kv_lora_rank (c_kv width)
D_R = 64        # rope width
D_QK = D_C + D_R  # 576: latent query / cache row width
TOPK = 2048     # index_topk
SCALE = 1.0 / 16.0  # 1/sqrt(qk_head_dim = 256)
N_PLANT = 64


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest-even), returned as uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Case:
    """One batch of query rows over a flat cache.

    Row i of the query tensors reads cache rows kv_start[i] .. kv_start[i]+n_vis[i]-1;
    its own key is the last of them (the query sees itself).
    """
    q_I: object          # [T,32,128] bf16 bits (uint16) or torch.bfloat16
    w: object            # [T,32]
    k_I: object          # [L,128]
    q: object            # [T,64,576]
    kv: object           # [L,576]
    kv_start: object     # [T] int64
    n_vis: object        # [T] int32
    plants: object       # [T,P] int32 positions relative to kv_start, -1 = none
    topk: int = TOPK
    name: str = ""
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.n_vis.shape[0])


# --------------------------------------------------------------------------
# plant-position laws (relative positions, self excluded)
# --------------------------------------------------------------------------

def _plants_uniform(rng, n_vis: int, p: int, lo_cap: int | None = None) -> np.ndarray:
    hi = n_vis - 1 if lo_cap is None else min(lo_cap, n_vis - 1)
    hi = max(hi, 0)
    m = min(p, hi)
    if m == 0:
        return np.zeros(0, np.int64)
    return rng.choice(hi, size=m, replace=False).astype(np.int64)


def _plants_loguniform(rng, n_vis: int, p: int, max_back: int, prefix_end: int) -> np.ndarray:
    """Distance back from the query log-uniform on [1, max_back], kept inside [0, prefix_end)."""
    t = n_vis - 1
    out: list[int] = []
    seen = set()
    tries = 0
    while len(out) < p and tries < 50 * p:
        tries += 1
        d = int(math.exp(rng.uniform(0.0, math.log(max_back + 1.0))))
        d = min(max(d, 1), max_back)
        s = t - d
        if s < 0 or s >= prefix_end or s in seen:
            continue
        seen.add(s)
        out.append(s)
    return np.asarray(out, np.int64)


# --------------------------------------------------------------------------
# numpy back end
# --------------------------------------------------------------------------

def make_case_numpy(seq_lens, queries, seed: int, n_plant: int = N_PLANT,
                    plant_law=None, topk: int = TOPK, name: str = "") -> Case:
    """Build a case.

    seq_lens : cache length of each sequence (sequences are laid out back to back).
    queries  : list of (seq_id, n_vis) — one query row each, in row order.
    plant_law(rng, row, seq_id, n_vis) -> relative positions to plant for that row.
    """
    rng = np.random.default_rng(seed)
    seq_lens = [int(x) for x in seq_lens]
    starts = np.zeros(len(seq_lens), np.int64)
    if len(seq_lens) > 1:
        starts[1:] = np.cumsum(seq_lens)[:-1]
    L = int(sum(seq_lens))
    T = len(queries)
    inv_sqrt_di = np.float32(1.0 / math.sqrt(D_I))

    q_I_f = (rng.standard_normal((T, H_I, D_I), dtype=np.float32) * inv_sqrt_di)
    q_I = bf16_from_f32(q_I_f)
    w = bf16_from_f32(rng.random((T, H_I), dtype=np.float32))
    k_I_f = rng.standard_normal((L, D_I), dtype=np.float32) * inv_sqrt_di
    q = bf16_from_f32(rng.standard_normal((T, H, D_QK), dtype=np.float32))
    kv = bf16_from_f32(rng.standard_normal((L, D_QK), dtype=np.float32))

    kv_start = np.array([starts[s] for s, _ in queries], np.int64)
    n_vis = np.array([nv for _, nv in queries], np.int32)
    for (s, nv) in queries:
        if not (1 <= nv <= seq_lens[s]):
            raise ValueError("n_vis must lie in [1, seq_len]")

    owner = np.full(L, -1, np.int64)
    if n_plant > 0:
        qf = bf16_to_f32(q_I)
        for i, (s, nv) in enumerate(queries):
            pos = (plant_law(rng, i, s, nv) if plant_law is not None
                   else _plants_uniform(rng, nv, n_plant))
            if pos.size == 0:
                continue
            u = qf[i].mean(axis=0)
            u = u / np.float32(np.linalg.norm(u) + 1e-30)
            noise = rng.standard_normal((pos.size, D_I), dtype=np.float32) * inv_sqrt_di
            rows = starts[s] + pos
            k_I_f[rows] = np.float32(0.8) * u[None, :] + np.float32(0.2) * noise
            owner[rows] = i
    k_I = bf16_from_f32(k_I_f)

    plants = np.full((T, max(n_plant, 1)), -1, np.int32)
    if n_plant > 0:
        rows = np.nonzero(owner >= 0)[0]
        fill = np.zeros(T, np.int64)
        for r in rows:
            i = int(owner[r])
            if fill[i] < plants.shape[1]:
                plants[i, fill[i]] = r - kv_start[i]
                fill[i] += 1
    return Case(q_I, w, k_I, q, kv, kv_start, n_vis, plants, topk, name)


# --------------------------------------------------------------------------
# named workloads (the five configurations the throughput claims are made on)
# --------------------------------------------------------------------------

def config3_lengths() -> np.ndarray:
    """Ragged decode context lengths: 32 draws uniform in [65536, 204800]."""
    return np.random.default_rng(0).integers(65536, 204800, endpoint=True, size=32)


WORKLOADS = {
    0: dict(name="decode_b4_ctx32k_shared", kind="decode"),
    1: dict(name="decode_b64_ctx128k", kind="decode"),
    2: dict(name="prefill_n32k", kind="prefill"),
    3: dict(name="decode_ragged_b32_ctx64k_200k", kind="decode"),
    4: dict(name="chunked_prefill_8k_over_1m", kind="prefill"),
}


def workload_layout(cfg: int, scale: int = 1):
    """(seq_lens, queries, plant kind) of a workload.

    ``scale`` > 1 shrinks every context length (and prefill query count) by that
    factor, giving a same-shaped case the oracle finishes in seconds.
    """
    if cfg == 0:
        L = 32768 // scale
        return [L], [(0, L)] * 4, "uniform"
    if cfg == 1:
        L = 131072 // scale
        return [L] * 64, [(b, L) for b in range(64)], "uniform"
    if cfg == 2:
        N = 32768 // scale
        return [N], [(0, t + 1) for t in range(N)], "uniform"
    if cfg == 3:
        lens = [int(x) // scale for x in config3_lengths()]
        return lens, [(b, lens[b]) for b in range(32)], "longrange"
    if cfg == 4:
        prefix = 1040384 // scale
        n_new = 8192 // scale
        return [prefix + n_new], [(0, prefix + i + 1) for i in range(n_new)], "loguniform"
    raise ValueError(cfg)


def _plant_law(kind: str, prefix_end: int | None, long_back: int):
    if kind == "uniform":
        return lambda rng, i, s, nv: _plants_uniform(rng, nv, N_PLANT)
    if kind == "longrange":
        def law(rng, i, s, nv):
            if i % 2 == 0:
                return _plants_uniform(rng, nv, N_PLANT, lo_cap=max(N_PLANT, nv - long_back))
            return _plants_uniform(rng, nv, N_PLANT)
        return law
    if kind == "loguniform":
        return lambda rng, i, s, nv: _plants_loguniform(rng, nv, N_PLANT, prefix_end, prefix_end)
    raise ValueError(kind)


def make_workload_numpy(cfg: int, scale: int = 1, seed: int | None = None) -> Case:
    seq_lens, queries, kind = workload_layout(cfg, scale)
    prefix_end = 1040384 // scale
    long_back = 100000 // scale
    law = _plant_law(kind, prefix_end, long_back)
    c = make_case_numpy(seq_lens, queries, cfg if seed is None else seed, plant_law=law,
                        name=WORKLOADS[cfg]["name"] + (f"/scale{scale}" if scale > 1 else ""))
    return c


# --------------------------------------------------------------------------
# torch back end (device-side generation for the multi-GB workloads)
# --------------------------------------------------------------------------

def make_workload_torch(cfg: int, device, scale: int = 1, seed: int | None = None,
                        chunk_rows: int = 1 << 20) -> Case:
    """Same recipe as ``make_workload_numpy`` drawn with a seeded torch generator
    on ``device``; tensors are torch (bf16 / int64 / int32) on that device."""
    import torch

    seq_lens, queries, kind = workload_layout(cfg, scale)
    prefix_end = 1040384 // scale
    long_back = 100000 // scale
    seed = cfg if seed is None else seed
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    rng = np.random.default_rng(seed)   # plant positions (host side, small)
    law = _plant_law(kind, prefix_end, long_back)

    starts = np.zeros(len(seq_lens), np.int64)
    if len(seq_lens) > 1:
        starts[1:] = np.cumsum(seq_lens)[:-1]
    L = int(sum(seq_lens))
    T = len(queries)
    inv = 1.0 / math.sqrt(D_I)

    def randn(shape, mul=1.0):
        return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * mul).to(torch.bfloat16)

    q_I = randn((T, H_I, D_I), inv)
    w = torch.rand((T, H_I), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    q = randn((T, H, D_QK))
    k_I = torch.empty((L, D_I), dtype=torch.bfloat16, device=device)
    kv = torch.empty((L, D_QK), dtype=torch.bfloat16, device=device)
    for r0 in range(0, L, chunk_rows):
        r1 = min(L, r0 + chunk_rows)
        k_I[r0:r1] = randn((r1 - r0, D_I), inv)
        kv[r0:r1] = randn((r1 - r0, D_QK))

    kv_start = torch.tensor([int(starts[s]) for s, _ in queries], dtype=torch.int64)
    n_vis = torch.tensor([nv for _, nv in queries], dtype=torch.int32)

    # plants: positions on the host, key rows built on the device, ascending row order
    rows_all, owners_all = [], []
    for i, (s, nv) in enumerate(queries):
        pos = law(rng, i, s, nv)
        if pos.size:
            rows_all.append(starts[s] + pos)
            owners_all.append(np.full(pos.size, i, np.int64))
    plants = np.full((T, N_PLANT), -1, np.int32)
    if rows_all:
        rows = np.concatenate(rows_all)
        owners = np.concatenate(owners_all)
        # last writer wins: keep, per row, the highest owner
        order = np.lexsort((owners, rows))
        rows, owners = rows[order], owners[order]
        last = np.ones(rows.size, bool)
        last[:-1] = rows[1:] != rows[:-1]
        rows, owners = rows[last], owners[last]
        u = q_I.float().mean(dim=1)
        u = u / (u.norm(dim=1, keepdim=True) + 1e-30)
        B = 1 << 18
        for b0 in range(0, rows.size, B):
            r = torch.from_numpy(rows[b0:b0 + B]).to(device)
            o = torch.from_numpy(owners[b0:b0 + B]).to(device)
            noise = torch.randn((r.numel(), D_I), generator=g, device=device, dtype=torch.float32) * inv
            k_I[r] = (0.8 * u[o] + 0.2 * noise).to(torch.bfloat16)
        fill = np.zeros(T, np.int64)
        for r, i in zip(rows, owners):
            if fill[i] < N_PLANT:
                plants[i, fill[i]] = r - int(starts[queries[i][0]])
                fill[i] += 1
    return Case(q_I, w, k_I, q, kv, kv_start.to(device), n_vis.to(device),
                plants, TOPK, WORKLOADS[cfg]["name"] + (f"/scale{scale}" if scale > 1 else ""))


def case_to_host(c: Case, rows=None) -> Case:
    """Copy a torch case to numpy uint16 / int arrays (optionally only some query rows).

    Cache tensors are copied whole; callers that need only a few sequences of a
    huge cache should slice before calling."""
    import torch

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    sel = slice(None) if rows is None else torch.as_tensor(rows, dtype=torch.long)
    ks = c.kv_start[sel] if rows is not None else c.kv_start
    return Case(u16(c.q_I[sel]), u16(c.w[sel]), u16(c.k_I), u16(c.q[sel]), u16(c.kv),
                ks.cpu().numpy().astype(np.int64), (c.n_vis[sel] if rows is not None else c.n_vis).cpu().numpy().astype(np.int32),
                c.plants[np.asarray(rows)] if rows is not None else c.plants, c.topk, c.name)


def make_shared_layer_torch(c: Case, layer: int, device, seed: int = 0, chunk_rows: int = 1 << 20):
    """Inputs of a further layer that shares ``c``'s indexer (IndexShare): its
    own queries q [T,64,576] and latent cache kv [rows,576], drawn like ``c``'s
    (N(0,1), bf16) from a seeded torch generator; the index set, kv_start and
    n_vis are the full layer's."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(1000003 * (layer + 1) + seed)
    q = torch.randn(tuple(c.q.shape), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    kv = torch.empty(tuple(c.kv.shape), dtype=torch.bfloat16, device=device)
    L = kv.shape[0]
    for r0 in range(0, L, chunk_rows):
        r1 = min(L, r0 + chunk_rows)
        kv[r0:r1] = torch.randn((r1 - r0, D_QK), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return q, kv


def make_shared_layer_numpy(c: Case, layer: int, seed: int = 0):
    """numpy (uint16 bf16 bits) counterpart of ``make_shared_layer_torch``."""
    r = np.random.default_rng(1000003 * (layer + 1) + seed)
    q = bf16_from_f32(r.standard_normal(c.q.shape).astype(np.float32))
    kv = bf16_from_f32(r.standard_normal(c.kv.shape).astype(np.float32))
    return q, kv

