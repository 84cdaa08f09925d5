"""Plant plausible mistakes in copies of the oracle source and check that the
pin suite fails on every one of them (the pins are not vacuous)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dsa_oracle.cpp")

MUTANTS = {
    "drop_rope_term": ("sc[j] = (nope + rope) * scale;", "sc[j] = nope * scale;"),
    "wrong_softmax_scale": ("sc[j] = (nope + rope) * scale;", "sc[j] = (nope + rope) * scale * 0.75;"),
    "no_normalisation": ("const double p = sc[j] / l;", "const double p = sc[j];"),
    "lse_sign": ("lse[h] = mx + std::log(l);", "lse[h] = mx - std::log(l);"),
    "tie_to_higher_position": ("return a < b;", "return a > b;"),
    "transposed_query_heads": ("dot += q[h * kIdxDim + d] * k[d];", "dot += q[d * kIdxHeads + h] * k[d];"),
    "single_head_weight": ("wh[h] = widen_bf16(w[h]);", "wh[h] = widen_bf16(w[0]);"),
    "excludes_self": ("int64_t keep = std::min<int64_t>(topk, n);", "int64_t keep = std::min<int64_t>(topk, n - 1);"),
    "rope_from_wrong_offset": ("rope += qh[kLatent + d] * r[kLatent + d];", "rope += qh[kLatent + d] * r[d];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mut = tmp_path / "mut.cpp"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["g++", "-O1", "-std=c++17", "-fPIC", "-shared", "-pthread", str(mut), "-o", str(so)])
    env = dict(os.environ, DSA_ORACLE_SO=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


# Plausible mistakes in the block-level variant (a Python front end over the same
# routines): each is planted in a copy of the oracle package, and the block pins
# must fail on it.
PY_SRC = os.path.join(ROOT, "oracle", "__init__.py")
BLOCK_MUTANTS = {
    "local_two_neighbours": ("LOCAL_SIDE = 1 ", "LOCAL_SIDE = 2 "),
    "anchor_last_block_of_16": ("for b in range(0, qb + 1, ANCHOR_EVERY)]", "for b in range(ANCHOR_EVERY - 1, qb + 1, ANCHOR_EVERY)]"),
    "block_score_mean": ("out.append(np.array([np.max(scores[i, b * BLOCK:min((b + 1) * BLOCK, n)])",
                         "out.append(np.array([np.mean(scores[i, b * BLOCK:min((b + 1) * BLOCK, n)])"),
    "block_ties_to_higher": ("key=lambda b: (-bsc[i][b], b))", "key=lambda b: (-bsc[i][b], -b))"),
    "drop_anchor_branch": ("o = sum(g[:, :, b, None] * outs[b] for b in range(3))",
                           "o = sum(g[:, :, b, None] * outs[b] for b in (0, 2))"),
    "dynamic_top_15": ("[:BLOCK_TOPK]", "[:BLOCK_TOPK - 1]"),
}


@pytest.mark.parametrize("name", ["unmutated"] + sorted(BLOCK_MUTANTS))
def test_block_pins_catch_mutant(name, tmp_path):
    old, new = BLOCK_MUTANTS.get(name, ("", ""))
    src = open(PY_SRC).read()
    assert name == "unmutated" or src.count(old) == 1, name
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text((src.replace(old, new) if old else src).replace(
        '_HERE = os.path.dirname(os.path.abspath(__file__))', '_HERE = %r' % os.path.join(ROOT, "oracle")))
    env = dict(os.environ, PYTHONPATH=str(tmp_path) + os.pathsep + ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-k", "block",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=600)
    assert "passed" in r.stdout or "failed" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
    if name == "unmutated":   # control: the copy itself passes, so a failure below is the mutation's
        assert r.returncode == 0, r.stdout[-2000:]
    else:
        assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"


# Plausible mistakes in the dense + sparse front end: the window shifted one
# position back (the query no longer sees itself), the gate applied to the wrong
# branch, the two branches' lse returned swapped.
DENSE_MUTANTS = {
    "window_shifted_back": ("p = n - window + np.arange(window", "p = n - window - 1 + np.arange(window"),
    "gate_on_sparse_branch": ("return g * o_d + (1.0 - g) * o_s, lse_d, lse_s",
                              "return g * o_s + (1.0 - g) * o_d, lse_d, lse_s"),
    "branch_lse_swapped": ("return g * o_d + (1.0 - g) * o_s, lse_d, lse_s",
                           "return g * o_d + (1.0 - g) * o_s, lse_s, lse_d"),
}


@pytest.mark.parametrize("name", ["unmutated"] + sorted(DENSE_MUTANTS))
def test_dense_sparse_pins_catch_mutant(name, tmp_path):
    old, new = DENSE_MUTANTS.get(name, ("", ""))
    src = open(PY_SRC).read()
    assert name == "unmutated" or src.count(old) == 1, name
    pkg = tmp_path / "oracle"
    pkg.mkdir()
    (pkg / "__init__.py").write_text((src.replace(old, new) if old else src).replace(
        '_HERE = os.path.dirname(os.path.abspath(__file__))', '_HERE = %r' % os.path.join(ROOT, "oracle")))
    env = dict(os.environ, PYTHONPATH=str(tmp_path) + os.pathsep + ROOT)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", "-k", "dense_sparse",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=str(tmp_path), env=env, capture_output=True, text=True, timeout=600)
    assert "passed" in r.stdout or "failed" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]
    if name == "unmutated":
        assert r.returncode == 0, r.stdout[-2000:]
    else:
        assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
