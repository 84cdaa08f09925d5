"""Benchmark of the DSA sparse-attention step (indexer -> top-k -> sparse MLA).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config C] [--scale S] [--skip-cpu] [--skip-e2e] [--e2e-serial]
                    [--workloads auto|none|LIST] [--no-graph] [--indexshare L]
                    [--dense-window W] [--block-sparse]

One step = one dsa_forward over one batch of the workload (every query row:
indexer over its causal context, exact top-2048, sparse latent MLA).  The
default workload is batch-64 decode at 131072 context per sequence.  Inputs
are synthetic (seeded) and resident in HBM; the default per-step working set
(about 2.3 GB) is far larger than the 126 MB L2, so no L2 flush is needed
between its steps (a workload whose inputs fit in L2 is flushed before every
timed step and its steps are timed one by one).  The line's `workloads` key
carries the other workloads, each timed for about a second.  Under torchrun
every rank runs its own batch (weak scaling; the path has no data exchange
between rows).  Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle on the same workload shape
(rank 0 only; bounded samples of query rows per step).

``--indexshare L`` times an IndexShare group instead: one step runs the full
layer (dsa_forward) and L-1 layers that reuse its index set
(dsa_sparse_mla_attn with their own queries and latent caches); the line
adds the full-layer and shared-layer times.  ``--dense-window W`` times the
dense + sparse layer: the selection, then dsa_dense_sparse_attn (attention over
the selected set and over the last W positions, fused per head).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from indexer_selected_sparse_dsa_b200 import workloads as wl  # noqa: E402

METRIC_DECODE = "decode tokens/s"
METRIC_PREFILL = "prefill query-tokens/s"
TOPK = wl.TOPK
L2_BYTES = 126 << 20      # B200 L2
FLUSH_BYTES = 256 << 20   # a write larger than L2 evicts every input line


def metric_for(cfg):
    return METRIC_DECODE if wl.WORKLOADS[cfg]["kind"] == "decode" else METRIC_PREFILL


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, source="fallback")


# ----------------------------------------------------------------------------- work model

def work_model(n_vis: np.ndarray, kv_start: np.ndarray, topk: int = TOPK):
    """Algorithmic bytes and flops of one step, per component (the units the
    roofline fractions use).  Key rows shared by several query rows (same
    kv_start) are counted once: the ideal reads every cached key once."""
    n = n_vis.astype(np.float64)
    sel = np.minimum(n, topk)
    distinct_keys = 0.0
    for ks in np.unique(kv_start):
        distinct_keys += float(n[kv_start == ks].max())
    q_idx = 32 * 128 * 2 + 32 * 2                       # q_I + w per row
    idx_bytes = 256 * distinct_keys + (4 * n + q_idx).sum()   # keys once, scores written
    idx_flops = (2 * 32 * 128 * n).sum()                # 32-head form
    topk_bytes = (4 * n).sum() + 4 * topk * n.size      # scores read, indices written
    # a selected latent row leaves DRAM once however many rows select it
    gathered = 1152 * min(float(sel.sum()), distinct_keys)
    per_row_io = 64 * 576 * 2 + 64 * 512 * 4 + 64 * 4       # q in, o_lat and lse out
    att_bytes = gathered + (per_row_io + 4 * topk) * n.size
    att_flops = (2 * 64 * sel * (576 + 512)).sum()
    step_bytes = 256 * distinct_keys + gathered + (q_idx + per_row_io) * n.size
    return dict(indexer_bytes=idx_bytes, indexer_flops=idx_flops, topk_bytes=topk_bytes, topk_flops=0.0,
                attention_bytes=att_bytes, attention_flops=att_flops, step_bytes=step_bytes,
                step_flops=idx_flops + att_flops)


def roofline_of(name, ms, nbytes, flops, pk, traffic=None):
    """Bound by arithmetic intensity against the ridge point; tensor peaks are
    the sustained figure (these kernels run inside a long step)."""
    gbs = nbytes / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    ridge = pk["bf16_sust"] * 1e12 / (pk["hbm"] * 1e9)
    if flops > 0 and flops / max(nbytes, 1.0) > ridge:
        return {"kernel": name, "bound": "tensor", "achieved": round(tfs, 1), "peak": pk["bf16_sust"],
                "unit": "TFLOP/s", "frac": round(tfs / pk["bf16_sust"], 4),
                "peak_source": pk["source"] + " (bf16 sustained)", "traffic": traffic,
                "algorithmic_flops_per_launch": float(flops), "algorithmic_bytes_per_launch": float(nbytes),
                "launch_ms": round(ms, 4)}
    return {"kernel": name, "bound": "hbm", "achieved": round(gbs, 1), "peak": pk["hbm"], "unit": "GB/s",
            "frac": round(gbs / pk["hbm"], 4), "peak_source": pk["source"] + " (HBM copy)", "traffic": traffic,
            "algorithmic_bytes_per_launch": float(nbytes), "algorithmic_flops_per_launch": float(flops),
            "launch_ms": round(ms, 4)}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None, interval_ms: int = 50):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", str(interval_ms)]
        if bus_id:
            cmd += ["-i", bus_id]
        try:
            self.p = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.p = None
        self.lines: list[str] = []

    def stop(self):
        if self.p is None:
            return
        time.sleep(0.12)
        self.p.terminate()
        try:
            out, _ = self.p.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
            out, _ = self.p.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


def bus_id_of(dev):
    import torch
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
    except Exception:
        return None


# ----------------------------------------------------------------------------- profiles

def lib_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "indexer_selected_sparse_dsa_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the
    current kernel sources (same source hash); else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d[f"{kernel}/{workload}"]
        if e.get("source_hash") == lib_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


# ----------------------------------------------------------------------------- ranks

def reduce_max_ms(ms: float, dist, device) -> float:
    """Max of a per-rank time over all ranks (every rank calls this)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(rows_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units of all ranks per second, timed by the slowest rank."""
    return rows_per_rank * world / (ms_per_step * 1e-3)


def forward_streams(T: int, max_n: int) -> bool:
    """dsa_forward's rule: stream scores into the selector when the score matrix
    would exceed 8 GB."""
    mode = os.environ.get("DSA_FORWARD_MODE")
    if mode in ("stream", "materialize"):
        return mode == "stream"
    return T * ((max_n + 3) // 4 * 4) * 4 > (8 << 30)


def launches_per_step(T: int, k: int, streams: bool, sms: int) -> int:
    """Kernels of this library one dsa_forward launches: indexer plan, indexer,
    top-k (materialised path) or the redo plan, the redo sweep and the buffer
    selection (streamed path), attention, and the split merge when rows are
    split over several CTAs."""
    ntiles = (k + 127) // 128
    splits = max(1, min(16, ntiles, sms // max(T, 1)))
    return 2 + (3 if streams else 1) + 1 + (1 if splits > 1 else 0)


def attention_launches(T: int, k: int, sms: int) -> int:
    """Kernels one dsa_sparse_mla_attn launches: attention, and the split merge."""
    ntiles = (k + 127) // 128
    return 1 + (1 if max(1, min(16, ntiles, sms // max(T, 1))) > 1 else 0)


def rank_seed(cfg: int, rank: int) -> int:
    """Each rank draws its own replica batch (weak scaling)."""
    return cfg + 7919 * rank


# ----------------------------------------------------------------------------- our arm

def extra_workloads(args, world):
    """Workloads measured after the headline one, each into the line's
    ``workloads`` key: by default (one GPU, plain step, full size) all the
    other four, so one run carries both halves of the metric."""
    if args.workloads == "none":
        return []
    if args.workloads == "auto":
        if world != 1 or args.scale != 1 or args.indexshare > 1 or args.dense_window > 0 or args.block_sparse:
            return []
        return [c for c in (0, 1, 2, 3, 4) if c != args.config]
    return [int(x) for x in args.workloads.split(",") if x.strip() and int(x) != args.config]


def run_ours(args, rank, world, dist):
    import torch
    from indexer_selected_sparse_dsa_b200 import binding as B
    from indexer_selected_sparse_dsa_b200 import build

    build.build()
    B.lib()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    out = measure(args.config, args.steps, args, dev, rank, world, dist, headline=True)
    extras = extra_workloads(args, world)
    if extras:
        out["workloads"] = {}
        for cfg in extras:
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
            r = measure(cfg, None, args, dev, rank, world, dist, headline=False)
            out["workloads"][r["config"]["workload"]] = r
            out["gpu_launches"] += r["gpu_launches"]
    if rank == 0:
        print(json.dumps(out), flush=True)


def measure(cfg, steps, args, dev, rank, world, dist, headline):
    """One workload: W warm-up steps, then `steps` timed steps (None: enough
    steps for at least about one second of timed region), the per-kernel
    breakdown, the roofline figures and, on rank 0 of a one-GPU run, the oracle
    on a bounded sample of the same rows.  The headline workload also carries
    the IndexShare / dense + sparse modes and the end-to-end leg."""
    import torch
    from indexer_selected_sparse_dsa_b200 import binding as B

    scale = args.scale
    c = wl.make_workload_torch(cfg, dev, scale=scale, seed=rank_seed(cfg, rank))
    T = c.T
    n_vis_h = c.n_vis.cpu().numpy()
    max_n = int(n_vis_h.max())
    k = TOPK
    o = torch.empty((T, 64, 512), dtype=torch.float32, device=dev)
    lse = torch.empty((T, 64), dtype=torch.float32, device=dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    ws = B.workspace(B.DSA_OP_FORWARD, T, max_n, k, device=dev)
    # a stream of our own: the timed steps can be captured into a CUDA graph on it
    torch.cuda.synchronize(dev)
    stream = torch.cuda.Stream(dev)

    # IndexShare (N^2, section "IndexShare"): a group of L layers runs the indexer
    # and the top-k once (the full layer) and L - 1 shared layers attend over the
    # same index set with their own queries and latent caches.
    L = max(1, args.indexshare) if headline else 1
    shared = [wl.make_shared_layer_torch(c, l, dev, seed=rank_seed(cfg, rank)) for l in range(1, L)]
    mla_ws = B.workspace(B.DSA_OP_SPARSE_MLA, T, max_n, k, device=dev)
    o_sh = [torch.empty_like(o) for _ in shared]
    lse_sh = [torch.empty_like(lse) for _ in shared]

    def full_layer():
        B.dsa_forward(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, max_n, k, wl.SCALE, o, lse, idx, ws, stream)

    # Dense + sparse ("GLM-5.2's DSA architecture: how dense and sparse attention
    # split the work", section "DSA's core design"): the selection, then both
    # attention branches (window of W positions, selected set) fused per head.
    # Block-level variant ("GLM-5: 744B parameters, 202K long context", section 2):
    # local, anchor and top-16-block branches over 128-token blocks, fused per head.
    BS = args.block_sparse and headline
    if BS:
        gates_b = torch.full((T, 64, 3), 1.0 / 3.0, dtype=torch.float32, device=dev)  # the caller's weights
        ws_b = B.workspace(B.DSA_OP_BLOCK_SPARSE, T, max_n, 0, device=dev)

        def block_layer():
            B.dsa_block_sparse_attn(c.q_I, c.w, c.k_I, c.q, c.kv, c.kv_start, c.n_vis, max_n, gates_b, wl.SCALE, o,
                                    None, None, ws_b, stream)
    W = args.dense_window if headline else 0
    if W > 0:
        gate = torch.full((T, 64), 0.5, dtype=torch.float32, device=dev)   # the caller's fusion weights
        ds_ws = B.workspace(B.DSA_OP_DENSE_SPARSE, T, 0, 0, device=dev)
        if forward_streams(T, max_n):
            sel_ws0 = B.workspace(B.DSA_OP_INDEXER_TOPK, T, max_n, k, device=dev)

            def select():
                B.dsa_indexer_topk(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, max_n, k, idx, sel_ws0, stream)
        else:
            plan_ws0 = B.workspace(B.DSA_OP_INDEXER, T, max_n, k, device=dev)
            scores0 = torch.empty((T, (max_n + 3) // 4 * 4), dtype=torch.float32, device=dev)

            def select():
                B.dsa_indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, scores0, plan_ws0, stream)
                B.dsa_topk(scores0, c.n_vis, k, idx, stream)

        def dense_sparse():
            B.dsa_dense_sparse_attn(c.q, c.kv, c.kv_start, c.n_vis, idx, W, gate, wl.SCALE, o, None, None, ds_ws,
                                    stream)

    def step():
        if BS:
            block_layer()
            return
        if W > 0:
            select()
            dense_sparse()
            return
        full_layer()
        for (q_l, kv_l), o_l, lse_l in zip(shared, o_sh, lse_sh):
            B.dsa_sparse_mla_attn(q_l, kv_l, c.kv_start, idx, wl.SCALE, o_l, lse_l, mla_ws, stream)

    for _ in range(args.warmup):
        step()
    B.dsa_sync_status(stream)
    if steps is None:
        # enough steps for about a second of timed region (at least 10)
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(3):
            step()
        torch.cuda.synchronize(dev)
        est_ms = max((time.perf_counter() - t0) * 1e3 / 3, 1e-3)
        steps = int(min(20000, max(10, math.ceil(1000.0 / est_ms))))

    # One step captured as a CUDA graph (the library's calls only enqueue kernels
    # and memsets on the stream), replayed K times: no host launch gaps.
    run, graph_note = step, None
    if args.graph:
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g, stream=stream):
                    step()
            torch.cuda.synchronize(dev)
            run = g.replay
        except Exception as e:  # capture refused: time the eager launches instead
            torch.cuda.synchronize(dev)
            graph_note = f"eager launches (graph capture failed: {type(e).__name__})"
    torch.cuda.synchronize(dev)

    # ---- timed region: exactly K steps
    # Inputs that fit in L2 would stay there from one step to the next: then L2 is
    # flushed (a 256 MB write) before every timed step and the steps are timed one
    # by one, the flush outside each step's events.
    in_bytes = sum(int(t.numel()) * t.element_size() for t in (c.q_I, c.w, c.k_I, c.q, c.kv))
    flush_l2 = in_bytes < 2 * L2_BYTES
    fbuf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush_l2 else None
    sampler = ClockSampler(bus_id_of(dev))
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if flush_l2:
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        with torch.cuda.stream(stream):
            for a0, a1 in pairs:
                fbuf.zero_()
                a0.record(stream)
                run()
                a1.record(stream)
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
        ms = sum(a0.elapsed_time(a1) for a0, a1 in pairs)
    else:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for _ in range(steps):
                run()
            ev1.record(stream)
        torch.cuda.synchronize(dev)
        if dist:
            dist.barrier()
        ms = ev0.elapsed_time(ev1)
    B.dsa_sync_status(stream)
    ms = reduce_max_ms(ms, dist, dev)
    sampler.stop()
    clocks = sampler.summary()
    if clocks is None or clocks["samples"] < 3:
        # timed region shorter than the sampling interval: sample an equal-load loop
        s2 = ClockSampler(bus_id_of(dev))
        t_end = time.time() + 1.0
        with torch.cuda.stream(stream):
            while time.time() < t_end:
                for _ in range(20):
                    run()
                torch.cuda.synchronize(dev)
        s2.stop()
        clocks = s2.summary()
        if clocks is not None:
            clocks["note"] = "sampled during an equal-load loop right after the timed region (timed region too short)"
    ms_step = ms / steps

    # ---- per-kernel breakdown: the same kernels dsa_forward runs, through the component
    # entry points, with CUDA events between them on the launching stream
    streams = forward_streams(T, max_n)
    nb = max(3, min(steps, 50))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nb)]
    wm = work_model(n_vis_h, c.kv_start.cpu().numpy())
    pk = peaks()
    workload = wl.WORKLOADS[cfg]["name"] + (f"_scale{scale}" if scale > 1 else "")
    if streams:
        sel_ws = B.workspace(B.DSA_OP_INDEXER_TOPK, T, max_n, k, device=dev)
    else:
        plan_ws = B.workspace(B.DSA_OP_INDEXER, T, max_n, k, device=dev)
        ld = (max_n + 3) // 4 * 4
        scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    torch.cuda.synchronize(dev)
    for e in evs:
        if flush_l2:
            with torch.cuda.stream(stream):
                fbuf.zero_()
        e[0].record(stream)
        if streams:
            B.dsa_indexer_topk(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, max_n, k, idx, sel_ws, stream)
            e[1].record(stream)
        else:
            B.dsa_indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, scores, plan_ws, stream)
            e[1].record(stream)
            B.dsa_topk(scores, c.n_vis, k, idx, stream)
        e[2].record(stream)
        B.dsa_sparse_mla_attn(c.q, c.kv, c.kv_start, idx, wl.SCALE, o, lse, mla_ws, stream)
        e[3].record(stream)
    torch.cuda.synchronize(dev)
    B.dsa_sync_status(stream)
    t_idx = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_topk = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    t_att = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    att = roofline_of("sparse MLA (dsa_sparse_mla_attn: split CTAs + merge)", t_att, wm["attention_bytes"],
                      wm["attention_flops"], pk, profiled_traffic("sparse_mla", workload))
    if streams:
        sel_bytes = wm["indexer_bytes"] - 4 * float(n_vis_h.sum()) + 4 * k * T   # no score matrix, indices out
        per_kernel = {
            "indexer_topk": roofline_of("indexer + streamed top-k (dsa_indexer_topk: plan + tcgen05 kernel)",
                                        t_idx, sel_bytes, wm["indexer_flops"], pk,
                                        profiled_traffic("indexer_topk", workload)),
            "sparse_mla": att,
        }
    else:
        per_kernel = {
            "indexer": roofline_of("indexer (dsa_indexer_scores: plan + tcgen05 kernel)", t_idx,
                                   wm["indexer_bytes"], wm["indexer_flops"], pk,
                                   profiled_traffic("indexer", workload)),
            "topk": roofline_of("top-k (dsa_topk)", t_topk, wm["topk_bytes"], 0.0, pk,
                                profiled_traffic("topk", workload)),
            "sparse_mla": att,
        }
    dominant = max(per_kernel, key=lambda kk: per_kernel[kk]["launch_ms"])
    roofline = per_kernel[dominant]
    kernels = {kk: {"ms": v["launch_ms"], "bound": v["bound"], "achieved": v["achieved"], "unit": v["unit"],
                    "frac": v["frac"]} for kk, v in per_kernel.items()}
    step_rf = roofline_of("dsa_forward step", ms_step, wm["step_bytes"], wm["step_flops"], pk)

    plain = (L == 1 and W == 0 and not BS)
    block_info = None
    if BS:
        nb = (max_n + 127) // 128
        block_info = {"block_tokens": 128, "dynamic_blocks": 16, "anchor_every_blocks": 16,
                      "local_positions": 384, "anchor_positions_max": ((nb + 15) // 16) * 128,
                      "gates": "1/3 per branch for every (row, head)", "block_layer_ms": round(ms_step, 4),
                      "token_step_breakdown": "the kernels and roofline of this line are the token-level step's"}
        workload += "_blocksparse"
    dense_info = None
    if W > 0:
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_t = max(3, min(steps, 200))
        a.record(stream)
        for _ in range(n_t):
            dense_sparse()
        b.record(stream)
        torch.cuda.synchronize(dev)
        B.dsa_sync_status(stream)
        dense_info = {"window": W, "gate": "0.5 for every (row, head)",
                      "dense_sparse_attention_ms": round(a.elapsed_time(b) / n_t, 4),
                      "sparse_attention_only_ms": round(t_att, 4)}
        workload += f"_dense{W}"
    indexshare = None
    if L > 1:
        # the full layer alone, and one shared layer's attention, timed the same way
        def timed(fn, n):
            torch.cuda.synchronize(dev)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            return a.elapsed_time(b) / n
        n_t = max(3, min(steps, 200))
        t_full = timed(full_layer, n_t)
        q1, kv1 = shared[0]
        t_shared = timed(lambda: B.dsa_sparse_mla_attn(q1, kv1, c.kv_start, idx, wl.SCALE, o_sh[0], lse_sh[0],
                                                      mla_ws, stream), n_t)
        B.dsa_sync_status(stream)
        indexshare = {"layers": L, "full_layers": 1, "shared_layers": L - 1, "group_ms": round(ms_step, 4),
                      "full_layer_ms": round(t_full, 4), "shared_layer_ms": round(t_shared, 4),
                      "shared_layer_tokens_per_s": round(whole_job_rate(T, world, t_shared), 1),
                      "unshared_group_ms_estimate": round(L * t_full, 4)}
        workload += f"_indexshare{L}"

    # ---- end to end through dsa_forward with host buffers
    e2e = None
    if headline and not args.skip_e2e and plain:
        e2e = run_e2e(args, c, o, lse, idx, ws, max_n, k, dev, stream, dist)
        if e2e is not None:
            e2e["value"] = round(whole_job_rate(T, world, e2e.pop("ms_per_step")), 1)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu and plain:
        cpu = cpu_baseline(c, o, lse, idx, cfg, budget_s=15.0 if headline else 6.0)

    value = whole_job_rate(T, world, ms_step)
    out = {
        "metric": metric_for(cfg), "value": round(value, 1),
        "unit": "tokens/s" if metric_for(cfg) == METRIC_DECODE else "query-tokens/s",
        "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload, "batch_rows": T, "max_context": max_n, "topk": k,
                   "indexer_heads": 32, "indexer_dim": 128, "mla_heads": 64, "kv_lora_rank": 512, "rope_dim": 64,
                   "l2": ("L2 flushed before every timed step (256 MB write; the inputs fit in L2), steps timed "
                          "one by one" if flush_l2 else "inputs larger than L2 (no flush)"),
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "step_roofline": {kk: step_rf[kk] for kk in ("bound", "achieved", "peak", "unit", "frac",
                                                     "algorithmic_bytes_per_launch", "algorithmic_flops_per_launch")},
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": (launches_per_step(T, k, streams, torch.cuda.get_device_properties(dev).multi_processor_count)
                         + (L - 1) * attention_launches(T, k, torch.cuda.get_device_properties(dev).multi_processor_count))
        * steps,
        "clocks": clocks,
        "launch": graph_note or (f"one CUDA graph per step (captured {'dsa_block_sparse_attn' if BS else 'dsa_forward'})"
                                 if args.graph else "eager launches"),
    }
    if indexshare is not None:
        out["indexshare"] = indexshare
    if block_info is not None:
        out["block_sparse"] = block_info
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # plan, indexer, block scores, block top-k, index lists, 3 x attention (+ merges), fusion
        out["gpu_launches"] = (2 + 1 + 1 + 1 + attention_launches(T, 384, sms) + attention_launches(T, 2048, sms)
                               + attention_launches(T, block_info["anchor_positions_max"], sms) + 1) * steps
    if dense_info is not None:
        out["dense_sparse"] = dense_info
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        # dsa_forward's kernels (its attention is the sparse branch), the dense branch, window indices, fusion
        out["gpu_launches"] = (launches_per_step(T, k, streams, sms) + attention_launches(T, W, sms) + 2) * steps
    if not headline:
        for key in ("n_gpus", "scaling", "vs_baseline", "data", "dtype", "e2e", "higher_is_better"):
            out.pop(key, None)
    return out


def run_e2e(args, c, o, lse, idx, ws, max_n, k, dev, stream, dist):
    """dsa_forward with the step's inputs copied in from pinned host memory and
    its result copied out, every step.  The cache stays resident (it is state
    that persists across decode steps); the rows this step appends to it (the
    new token's k_I and latent row of each sequence) are part of the copy-in.

    Pipelined (default): two sets of input and output buffers; step i + 1's
    copy-in (one copy stream) and step i - 1's copy-out (another) run while
    step i computes, as a serving loop would.  --e2e-serial runs copy-in,
    compute and copy-out of each step back to back on one stream instead."""
    import torch
    from indexer_selected_sparse_dsa_b200 import binding as B
    serial = args.e2e_serial
    nb = 1 if serial else 2
    new_rows = (c.kv_start + c.n_vis.to(torch.int64) - 1)
    h = {
        "q_I": c.q_I.cpu().pin_memory(), "w": c.w.cpu().pin_memory(), "q": c.q.cpu().pin_memory(),
        "kv_start": c.kv_start.cpu().pin_memory(), "n_vis": c.n_vis.cpu().pin_memory(),
        "k_new": c.k_I[new_rows].cpu().pin_memory(), "kv_new": c.kv[new_rows].cpu().pin_memory(),
        "rows": new_rows.cpu().pin_memory(),
    }
    d = [{kk: torch.empty_like(v, device=dev) for kk, v in h.items()} for _ in range(nb)]
    o_d = [o] + [torch.empty_like(o) for _ in range(nb - 1)]
    lse_d = [lse] + [torch.empty_like(lse) for _ in range(nb - 1)]
    o_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(nb)]
    lse_h = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(nb)]
    bi = sum(v.numel() * v.element_size() for v in h.values())
    bo = o_h[0].numel() * 4 + lse_h[0].numel() * 4
    cin, cout = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(nb)]    # buffer set b: inputs landed
    ev_done = [torch.cuda.Event() for _ in range(nb)]  # buffer set b: step computed (inputs consumed)
    ev_out = [torch.cuda.Event() for _ in range(nb)]   # buffer set b: outputs copied out

    def compute(b):
        c.k_I.index_copy_(0, d[b]["rows"], d[b]["k_new"])
        c.kv.index_copy_(0, d[b]["rows"], d[b]["kv_new"])
        B.dsa_forward(d[b]["q_I"], d[b]["w"], c.k_I, d[b]["q"], c.kv, d[b]["kv_start"], d[b]["n_vis"], max_n, k,
                      wl.SCALE, o_d[b], lse_d[b], idx, ws, stream)

    def step(i):
        b = i % nb
        if serial:
            with torch.cuda.stream(stream):   # copies, cache update and dsa_forward in one stream order
                for kk in h:
                    d[b][kk].copy_(h[kk], non_blocking=True)
                compute(b)
                o_h[b].copy_(o_d[b], non_blocking=True)
                lse_h[b].copy_(lse_d[b], non_blocking=True)
            return
        with torch.cuda.stream(cin):
            cin.wait_event(ev_done[b])        # the step that last used set b has read its inputs
            for kk in h:
                d[b][kk].copy_(h[kk], non_blocking=True)
            ev_in[b].record(cin)
        with torch.cuda.stream(stream):
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])      # set b's previous outputs have left the device
            compute(b)
            ev_done[b].record(stream)
        with torch.cuda.stream(cout):
            cout.wait_event(ev_done[b])
            o_h[b].copy_(o_d[b], non_blocking=True)
            lse_h[b].copy_(lse_d[b], non_blocking=True)
            ev_out[b].record(cout)

    def run(n):
        for i in range(n):
            step(i)
        stream.wait_stream(cout)              # the last copy-out is part of the run

    run(max(3, args.warmup))
    torch.cuda.synchronize(dev)
    steps = args.steps
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cin.wait_stream(stream)                   # the first copy-in starts inside the timed region
    run(steps)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    ms = reduce_max_ms(e0.elapsed_time(e1), dist, dev)
    B.dsa_sync_status(stream)
    # every step computes the same batch: each buffer set's copied-out result must
    # equal the device-resident run's (the kernels are deterministic)
    same = all(torch.equal(o_h[b], o_d[0].cpu()) and torch.equal(lse_h[b], lse_d[0].cpu()) for b in range(nb))
    return {"ms_per_step": ms / steps, "unit": "tokens/s" if metric_for(args.config) == METRIC_DECODE else "query-tokens/s",
            "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo), "api": "dsa_forward",
            "mode": "serial" if serial else "pipelined: step i+1 copy-in and step i-1 copy-out overlap step i",
            "outputs_match_device_run": bool(same)}


def host_rows(c, rows):
    """Host copies (uint16 bf16 bits) of some query rows of a device case and of
    only their visible cache prefixes; rows of one sequence share one copy."""
    import torch

    def u16(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    ks = c.kv_start[rows].cpu().numpy()
    nv = c.n_vis[rows].cpu().numpy()
    longest = {}
    for s0, n in zip(ks, nv):
        longest[int(s0)] = max(longest.get(int(s0), 0), int(n))
    kI, kv, base, off = [], [], {}, 0
    for s0, n in longest.items():
        kI.append(u16(c.k_I[s0:s0 + n]))
        kv.append(u16(c.kv[s0:s0 + n]))
        base[s0] = off
        off += n
    starts = np.array([base[int(s0)] for s0 in ks], np.int64)
    return (u16(c.q_I[rows]), u16(c.w[rows]), np.concatenate(kI), u16(c.q[rows]), np.concatenate(kv), starts,
            nv.astype(np.int32))


def sample_rows(T: int, n: int):
    """n query rows spread over a batch, the last (longest) row included."""
    if n >= T:
        return list(range(T))
    return sorted({int(x) for x in np.linspace(0, T - 1, n).round()})


def cpu_baseline(c, o, lse, idx, cfg, budget_s: float = 15.0):
    """The oracle, as it stands, on the host cores over a bounded sample of this
    run's own query rows (their caches copied back), one row per core per
    call; also reports how far the GPU's outputs for those rows are from the
    oracle's."""
    import oracle
    cores = os.cpu_count() or 1
    T = c.T
    order = list(range(T)) if wl.WORKLOADS[cfg]["kind"] == "decode" else sample_rows(T, 16 * cores)
    rows_done, t_spent, maxerr = 0, 0.0, 0.0
    while rows_done < len(order) and t_spent < budget_s:
        rows = order[rows_done:rows_done + cores]
        q_I, w, kI, q, kv, starts, nv = host_rows(c, rows)
        t0 = time.perf_counter()
        o_ref, lse_ref, idx_ref = oracle.forward(q_I, w, kI, q, kv, starts, nv, TOPK, wl.SCALE, nthreads=cores)
        t_spent += time.perf_counter() - t0
        rows_done += len(rows)
        g = o[rows].cpu().numpy().astype(np.float64)
        maxerr = max(maxerr, float(np.max(np.abs(g - o_ref))))
    unit = "tokens/s" if metric_for(cfg) == METRIC_DECODE else "query-tokens/s"
    what = "query rows of this run" if wl.WORKLOADS[cfg]["kind"] == "decode" else "query rows spread over this run's batch"
    return {"value": round(rows_done / t_spent, 3), "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{rows_done} of {T} {what} (full causal context each, {cores} rows per call), "
                      f"fp64 C++ oracle, {t_spent:.1f} s",
            "gpu_vs_oracle_max_abs_on_sample": maxerr}


# ----------------------------------------------------------------------------- reference arm

def reference_case(cfg: int, scale: int, rows: int):
    """A bounded host-side sample of workload `cfg` for the oracle: `rows` query
    rows with the workload's own context lengths.  Decode rows query one shared
    cache of the workload's context length (the oracle's work per row is the
    same as over a cache of its own; one cache keeps host memory bounded);
    prefill rows are the last rows of the workload's batch (the longest
    contexts)."""
    seq_lens, queries, _kind = wl.workload_layout(cfg, scale)
    if wl.WORKLOADS[cfg]["kind"] == "decode":
        picked = [queries[j % len(queries)] for j in range(rows)]
        L = max(n for _, n in picked)
        return wl.make_case_numpy([L], [(0, n) for _, n in picked], seed=cfg)
    return wl.make_case_numpy(seq_lens, queries[-rows:], seed=cfg)


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    cores = os.cpu_count() or 1
    cfg, scale = args.config, args.scale
    c = reference_case(cfg, scale, cores)
    rows_per_step = min(c.T, cores)           # one row per core per step
    budget = 150.0
    times, rows_total = [], 0
    t_start = time.perf_counter()
    steps_done = 0
    r = 0
    for s in range(args.warmup + args.steps):
        sel = [(r + j) % c.T for j in range(rows_per_step)]
        r += rows_per_step
        t0 = time.perf_counter()
        oracle.forward(c.q_I[sel], c.w[sel], c.k_I, c.q[sel], c.kv, c.kv_start[sel], c.n_vis[sel], TOPK, wl.SCALE,
                       nthreads=cores)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
            rows_total += len(sel)
            steps_done += 1
        if time.perf_counter() - t_start > budget and steps_done >= 1:
            break
    tot = sum(times)
    value = rows_total / tot
    unit = "tokens/s" if metric_for(cfg) == METRIC_DECODE else "query-tokens/s"
    workload = wl.WORKLOADS[cfg]["name"] + (f"_scale{scale}" if scale > 1 else "")
    seq_lens, queries, _ = wl.workload_layout(cfg, scale)
    out = {"impl": "reference", "metric": metric_for(cfg), "value": round(value, 4), "unit": unit, "n_gpus": world,
           "steps": steps_done, "steps_requested": args.steps, "warmup": args.warmup,
           "ms_per_step": round(1e3 * tot / max(steps_done, 1), 2), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": workload, "batch_rows": len(queries), "max_context": int(max(q[1] for q in queries)),
                      "topk": TOPK, "rows_per_step": rows_per_step},
           "cpu_baseline": {"kind": "oracle", "cores": cores, "value": round(value, 4), "unit": unit,
                            "sample": f"{rows_per_step} query rows per step, one per core, with the workload's "
                                      f"context lengths (full causal context each), fp64 C++ oracle, "
                                      f"{steps_done} steps in {tot:.1f} s"},
           "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=1, help="workload: 0..4 (default 1: decode b64 x 128K)")
    ap.add_argument("--scale", type=int, default=1, help="shrink contexts by this factor (small captures)")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--workloads", default="auto",
                    help="other workloads measured after the headline into the line's 'workloads' key: "
                         "'auto' (all others on one GPU at full size), 'none', or a comma list such as 2,4")
    ap.add_argument("--e2e-serial", action="store_true",
                    help="end-to-end leg: copy-in, compute and copy-out of each step back to back on one stream")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time eager launches instead of replaying the step captured as a CUDA graph")
    ap.add_argument("--dense-window", type=int, default=0,
                    help="time the dense + sparse layer instead: selection, then attention over the selected set "
                         "and over a window of W positions, fused per head (default 0: off)")
    ap.add_argument("--block-sparse", action="store_true",
                    help="time the block-level variant instead: 128-token blocks, local / anchor / top-16-block "
                         "branches fused per head (dsa_block_sparse_attn)")
    ap.add_argument("--indexshare", type=int, default=1,
                    help="layers per IndexShare group: one step = one full layer (indexer, top-k, attention) "
                         "+ L-1 layers attending over its index set (default 1: no sharing)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        run_ours(args, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
