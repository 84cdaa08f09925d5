"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, each with its own
replica batch (different seeds), max-over-ranks timing, whole-job rate."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from indexer_selected_sparse_dsa_b200 import workloads as wl
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank                         # a slower second rank
        m = bench.reduce_max_ms(ms, dist, "cpu")
        rate = bench.whole_job_rate(64, world, m)
        seq_lens, queries, _ = wl.workload_layout(1, scale=256)
        c = wl.make_case_numpy(seq_lens[:2], [q for q in queries if q[0] < 2], seed=bench.rank_seed(1, rank),
                               n_plant=2)
        out.put((rank, m, rate, int(c.k_I[:4].astype("int64").sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, v0, h0), (r1, m1, v1, h1) = res
    assert m0 == m1 == 15.0                      # every rank sees the slowest rank's time
    assert v0 == v1 == pytest.approx(64 * 2 / 15e-3)
    assert h0 != h1                              # distinct replica batches
