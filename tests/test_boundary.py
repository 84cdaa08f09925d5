"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

* the library loads and exports every function include/dsa.h declares;
* workspace sizes follow their stated rule;
* arguments that fail host validation are rejected before any CUDA call.
"""
import ctypes
import os
import re

import pytest

from indexer_selected_sparse_dsa_b200 import binding as B
from indexer_selected_sparse_dsa_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return B.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    return re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", src)


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    assert L.dsa_abi_version() == 1


def test_header_constants_match_config_table():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    consts = dict(re.findall(r"#define (DSA_\w+) (\d+)", src))
    assert consts["DSA_INDEX_HEADS"] == "32" and consts["DSA_INDEX_DIM"] == "128"
    assert consts["DSA_HEADS"] == "64" and consts["DSA_LATENT"] == "512" and consts["DSA_ROPE"] == "64"
    assert consts["DSA_ROW"] == "576" and consts["DSA_MAX_TOPK"] == "2048"


def test_workspace_sizes(L):
    def ws(op, T, n, k):
        return B.dsa_workspace_size(op, T, n, k)
    assert ws(B.DSA_OP_TOPK, 100, 1000, 2048) == 0
    assert ws(B.DSA_OP_INDEXER, 64, 131072, 0) % 256 == 0
    assert ws(B.DSA_OP_INDEXER, 64, 131072, 0) >= 32 + 64 * 32
    f = ws(B.DSA_OP_FORWARD, 64, 131072, 2048)
    assert f >= 64 * 131072 * 4 + 64 * 2048 * 4
    # score rows are padded to a multiple of 4 columns
    assert ws(B.DSA_OP_FORWARD, 3, 5, 8) >= 3 * 8 * 4
    assert ws(B.DSA_OP_FORWARD, -1, -1, -1) == ws(B.DSA_OP_FORWARD, 0, 0, 0)


def _err(rc, code):
    assert rc == code, (rc, B.last_error())
    assert B.last_error() != ""


def test_host_validation_rejects_bad_arguments(L):
    P = ctypes.c_void_p
    fake = P(1 << 20)            # never dereferenced: validation fails first
    odd = P((1 << 20) + 2)
    z = P(0)
    # T < 0
    _err(L.dsa_topk(fake, 8, fake, -1, 16, fake, z), B.DSA_ERR_INVALID_ARG)
    # topk out of range
    _err(L.dsa_topk(fake, 8, fake, 4, 0, fake, z), B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_topk(fake, 8, fake, 4, 2049, fake, z), B.DSA_ERR_INVALID_ARG)
    # score_ld not a multiple of 4
    _err(L.dsa_topk(fake, 6, fake, 4, 16, fake, z), B.DSA_ERR_INVALID_ARG)
    # null pointer
    _err(L.dsa_topk(z, 8, fake, 4, 16, fake, z), B.DSA_ERR_INVALID_ARG)
    # misaligned scores
    _err(L.dsa_topk(odd, 8, fake, 4, 16, fake, z), B.DSA_ERR_INVALID_ARG)
    # indexer: cache_rows out of range, missing workspace, workspace too small
    _err(L.dsa_indexer_scores(fake, fake, fake, 0, fake, fake, 4, fake, 8, fake, 1 << 20, z), B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_indexer_scores(fake, fake, fake, 1 << 31, fake, fake, 4, fake, 8, fake, 1 << 20, z), B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_indexer_scores(fake, fake, fake, 100, fake, fake, 4, fake, 8, z, 0, z), B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_indexer_scores(fake, fake, fake, 100, fake, fake, 4, fake, 8, fake, 16, z), B.DSA_ERR_WORKSPACE)
    _err(L.dsa_indexer_scores(fake, fake, odd, 100, fake, fake, 4, fake, 8, fake, 1 << 20, z), B.DSA_ERR_INVALID_ARG)
    # attention: bad scale, null o_lat
    _err(L.dsa_sparse_mla_attn(fake, fake, 100, fake, fake, 4, 16, ctypes.c_float(0.0), fake, z, z, 0, z),
         B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_sparse_mla_attn(fake, fake, 100, fake, fake, 4, 16, ctypes.c_float(0.0625), z, z, z, 0, z),
         B.DSA_ERR_INVALID_ARG)
    # forward: max_n_vis above cache_rows, workspace too small
    _err(L.dsa_forward(fake, fake, fake, fake, fake, 100, fake, fake, 4, 101, 16, ctypes.c_float(0.0625),
                       fake, z, z, fake, 1 << 30, z), B.DSA_ERR_INVALID_ARG)
    _err(L.dsa_forward(fake, fake, fake, fake, fake, 100, fake, fake, 4, 100, 16, ctypes.c_float(0.0625),
                       fake, z, z, fake, 256, z), B.DSA_ERR_WORKSPACE)
    # dense + sparse: window out of range, null gate, workspace too small
    ds = L.dsa_dense_sparse_attn
    for window in (0, 2049):
        _err(ds(fake, fake, 100, fake, fake, fake, 4, 16, window, fake, ctypes.c_float(0.0625), fake, z, z, fake,
                1 << 30, z), B.DSA_ERR_INVALID_ARG)
    _err(ds(fake, fake, 100, fake, fake, fake, 4, 16, 64, z, ctypes.c_float(0.0625), fake, z, z, fake, 1 << 30, z),
         B.DSA_ERR_INVALID_ARG)
    _err(ds(fake, fake, 100, fake, fake, fake, 4, 16, 64, fake, ctypes.c_float(0.0625), fake, z, z, fake, 256, z),
         B.DSA_ERR_WORKSPACE)


def test_empty_batch_is_a_no_op(L):
    z = ctypes.c_void_p(0)
    assert L.dsa_topk(z, 8, z, 0, 16, z, z) == B.DSA_OK
    assert L.dsa_indexer_scores(z, z, z, 10, z, z, 0, z, 8, z, 0, z) == B.DSA_OK
    assert L.dsa_sparse_mla_attn(z, z, 10, z, z, 0, 16, ctypes.c_float(0.0625), z, z, z, 0, z) == B.DSA_OK
    assert L.dsa_dense_sparse_attn(z, z, 10, z, z, z, 0, 16, 64, z, ctypes.c_float(0.0625), z, z, z, z, 0,
                                   z) == B.DSA_OK
