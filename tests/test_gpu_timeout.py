"""Hang protection of the device waits, tested without a fault.

Every spin-wait in the kernels has a time limit.  When it runs out the CTA
stops, lets the copies and tensor-core operations it started finish, releases
TMEM and exits; the call's status then reads DSA_ERR_TIMEOUT and the CUDA
context stays usable.  A child process (so the test process never shares a
context with an aborted kernel):
  1. runs the probe that waits on a barrier nothing completes: TIMEOUT;
  2. runs the attention, the indexer and the one-launch decode step (its
     grid-wide handoffs included) with a 1 ns limit (their first wait that is
     not already complete gives up): TIMEOUT, no CUDA error;
  3. restores the default limit and runs them again in the same process:
     status OK and the results match the oracle.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys
import numpy as np
import torch
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.join(ROOT, "tests"))
import oracle
from indexer_selected_sparse_dsa_b200 import binding as B, build, workloads as wl
from gpu_util import to_dev, assert_attention_close, assert_scores_close, assert_selection_ok

build.build()
out = {}

def status_of(fn):
    try:
        fn()
        B.dsa_sync_status()
        return "OK"
    except B.DSAError as e:
        return {B.DSA_ERR_TIMEOUT: "TIMEOUT", B.DSA_ERR_CUDA: "CUDA"}.get(e.code, str(e.code))

c = wl.make_case_numpy([6000, 3000], [(0, 6000), (0, 5999), (1, 3000), (1, 2500)], seed=11, n_plant=8)
d = to_dev(c)
T, k = c.T, 2048
ld = (int(c.n_vis.max()) + 3) // 4 * 4
idx = oracle.topk(oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, ld), c.n_vis, k)
idx_d = torch.from_numpy(idx).cuda()
o = torch.empty((T, 64, 512), device="cuda"); lse = torch.empty((T, 64), device="cuda")
scores = torch.empty((T, ld), device="cuda")
ws_i = B.workspace(B.DSA_OP_INDEXER, T, ld, 0)
ws_a = B.workspace(B.DSA_OP_SPARSE_MLA, T, 0, k)

def attention():
    B.dsa_sparse_mla_attn(d["q"], d["kv"], d["kv_start"], idx_d, wl.SCALE, o, lse, ws_a)

def indexer():
    B.dsa_indexer_scores(d["q_I"], d["w"], d["k_I"], d["kv_start"], d["n_vis"], scores, ws_i)

# the one-launch decode step (DSA_DECODE_FUSED=1): 3 rows over one 6000-position cache
cf = wl.make_case_numpy([6000], [(0, 6000), (0, 5999), (0, 3000)], seed=12)
df = to_dev(cf)
of = torch.empty((3, 64, 512), device="cuda"); lsef = torch.empty((3, 64), device="cuda")
idxf = torch.empty((3, k), dtype=torch.int32, device="cuda")
ws_f = B.workspace(B.DSA_OP_FORWARD, 3, 6000, k)

def fused():
    os.environ["DSA_DECODE_FUSED"] = "1"
    try:
        B.dsa_forward(df["q_I"], df["w"], df["k_I"], df["q"], df["kv"], df["kv_start"], df["n_vis"], 6000, k,
                      wl.SCALE, of, lsef, idxf, ws_f)
    finally:
        os.environ.pop("DSA_DECODE_FUSED", None)

B.dsa_set_wait_limit_ns(2_000_000)                 # 2 ms: the probe gives up quickly
out["probe"] = status_of(B.dsa_check_wait_timeout)
B.dsa_set_wait_limit_ns(1)
out["attention_1ns"] = status_of(attention)
out["indexer_1ns"] = status_of(indexer)
out["fused_1ns"] = status_of(fused)
B.dsa_set_wait_limit_ns(0)                         # default limit again, same context
out["attention_default"] = status_of(attention)
out["indexer_default"] = status_of(indexer)
out["fused_default"] = status_of(fused)
o_ref, lse_ref = oracle.sparse_mla(c.q, c.kv, c.kv_start, idx, wl.SCALE)
assert_attention_close(o.cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref)
S_ref = oracle.indexer_scores(c.q_I, c.w, c.k_I, c.kv_start, c.n_vis, ld)
assert_scores_close(scores.cpu().numpy(), S_ref, c.n_vis)
idx_h = idxf.cpu().numpy()
Sf = oracle.indexer_scores(cf.q_I, cf.w, cf.k_I, cf.kv_start, cf.n_vis, 6000)
assert_selection_ok(idx_h, Sf, cf.n_vis, k)
of_ref, lsef_ref = oracle.sparse_mla(cf.q, cf.kv, cf.kv_start, idx_h, wl.SCALE)
assert_attention_close(of.cpu().numpy(), lsef.cpu().numpy(), of_ref, lsef_ref)
out["parity_after"] = "OK"
print("RESULT " + json.dumps(out), flush=True)
'''


def test_bounded_waits_give_up_and_leave_the_context_usable():
    code = "import os\nROOT = %r\n" % ROOT + CHILD
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600, cwd=ROOT)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")]
    assert r.returncode == 0 and lines, f"child failed (rc {r.returncode}):\n{r.stdout[-3000:]}\n{r.stderr[-3000:]}"
    res = json.loads(lines[-1][len("RESULT "):])
    assert res["probe"] == "TIMEOUT", res
    assert res["attention_1ns"] == "TIMEOUT", res
    assert res["indexer_1ns"] == "TIMEOUT", res
    assert res["fused_1ns"] == "TIMEOUT", res
    assert res["attention_default"] == "OK" and res["indexer_default"] == "OK", res
    assert res["fused_default"] == "OK", res
    assert res["parity_after"] == "OK", res
