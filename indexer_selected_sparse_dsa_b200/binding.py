"""ctypes binding of libdsa (include/dsa.h): argument marshalling only.

Every function here takes torch tensors that already live on the current CUDA
device, checks dtypes and shapes, and passes raw pointers and sizes to the C
entry point of the same name.  All arithmetic happens in the CUDA kernels.
There is no fallback: if ``libdsa.so`` is missing or fails to load, every
call raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libdsa.so")

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, DSA_ERR_TIMEOUT, DSA_ERR_UNSUPPORTED, DSA_ERR_BAD_ROW = range(7)
(DSA_OP_INDEXER, DSA_OP_TOPK, DSA_OP_SPARSE_MLA, DSA_OP_FORWARD, DSA_OP_INDEXER_TOPK, DSA_OP_DENSE_SPARSE,
 DSA_OP_BLOCK_SPARSE) = range(7)
BLOCK_TOPK = 16
INDEX_HEADS, INDEX_DIM, HEADS, LATENT, ROPE, ROW, MAX_TOPK = 32, 128, 64, 512, 64, 576, 2048
NOALLOC_MAX_ROWS = 8192

_STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_WORKSPACE", 3: "DSA_ERR_CUDA",
                 4: "DSA_ERR_TIMEOUT", 5: "DSA_ERR_UNSUPPORTED", 6: "DSA_ERR_BAD_ROW"}


class DSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib():
    """Load libdsa.so (built in-tree).  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libdsa.so not built ({LIB_PATH}); run python -m indexer_selected_sparse_dsa_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        L.dsa_workspace_size.argtypes = [I, I, I64, I]
        L.dsa_workspace_size.restype = SZ
        L.dsa_indexer_scores.argtypes = [P, P, P, I64, P, P, I, P, I64, P, SZ, P]
        L.dsa_topk.argtypes = [P, I64, P, I, I, P, P]
        L.dsa_sparse_mla_attn.argtypes = [P, P, I64, P, P, I, I, F, P, P, P, SZ, P]
        L.dsa_forward.argtypes = [P, P, P, P, P, I64, P, P, I, I64, I, F, P, P, P, P, SZ, P]
        L.dsa_sync_status.argtypes = [P]
        L.dsa_indexer_topk.argtypes = [P, P, P, I64, P, P, I, I64, I, P, P, SZ, P]
        L.dsa_indexer_topk.restype = I
        L.dsa_indexer_scores_noalloc.argtypes = [P, P, P, I64, P, P, I, P, I64, P]
        L.dsa_dense_sparse_attn.argtypes = [P, P, I64, P, P, P, I, I, I, P, F, P, P, P, P, SZ, P]
        L.dsa_dense_sparse_attn.restype = I
        L.dsa_indexer_scores_noalloc.restype = I
        L.dsa_block_sparse_attn.argtypes = [P, P, P, P, P, I64, P, P, I, I64, P, F, P, P, P, P, SZ, P]
        L.dsa_block_sparse_attn.restype = I
        L.dsa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.dsa_set_wait_limit_ns.restype = None
        L.dsa_check_wait_timeout.argtypes = [P]
        L.dsa_check_wait_timeout.restype = I
        L.dsa_last_error_string.restype = ctypes.c_char_p
        L.dsa_abi_version.restype = I
        for name in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_mla_attn", "dsa_forward", "dsa_sync_status"):
            getattr(L, name).restype = I
        _lib = L
    return _lib


def last_error() -> str:
    return lib().dsa_last_error_string().decode()


def _check(rc: int):
    if rc != DSA_OK:
        raise DSAError(rc, last_error())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _need(t, dtype, shape=None, name=""):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def dsa_workspace_size(op: int, T: int, max_n_vis: int, topk: int) -> int:
    return int(lib().dsa_workspace_size(op, T, max_n_vis, topk))


def dsa_indexer_scores(q_I, w, k_I, kv_start, n_vis, scores, ws, stream=None):
    import torch
    T = n_vis.shape[0]
    _need(q_I, torch.bfloat16, (T, INDEX_HEADS, INDEX_DIM), "q_I")
    _need(w, torch.bfloat16, (T, INDEX_HEADS), "w")
    _need(k_I, torch.bfloat16, None, "k_I")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(scores, torch.float32, None, "scores")
    _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_indexer_scores(_ptr(q_I), _ptr(w), _ptr(k_I), k_I.shape[0], _ptr(kv_start), _ptr(n_vis), T,
                                    _ptr(scores), scores.shape[1], _ptr(ws), ws.numel(), _stream(stream)))


def dsa_indexer_scores_noalloc(q_I, w, k_I, kv_start, n_vis, scores, stream=None):
    """dsa_indexer_scores for callers that cannot allocate: no workspace; the
    library keeps the plan in its own fixed device array (at most
    NOALLOC_MAX_ROWS rows; calls must not overlap on the GPU)."""
    import torch
    T = n_vis.shape[0]
    _need(q_I, torch.bfloat16, (T, INDEX_HEADS, INDEX_DIM), "q_I")
    _need(w, torch.bfloat16, (T, INDEX_HEADS), "w")
    _need(k_I, torch.bfloat16, None, "k_I")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(scores, torch.float32, None, "scores")
    _check(lib().dsa_indexer_scores_noalloc(_ptr(q_I), _ptr(w), _ptr(k_I), k_I.shape[0], _ptr(kv_start),
                                            _ptr(n_vis), T, _ptr(scores), scores.shape[1], _stream(stream)))


def dsa_indexer_topk(q_I, w, k_I, kv_start, n_vis, max_n_vis, topk, idx, ws, stream=None):
    import torch
    T = n_vis.shape[0]
    _need(q_I, torch.bfloat16, (T, INDEX_HEADS, INDEX_DIM), "q_I")
    _need(w, torch.bfloat16, (T, INDEX_HEADS), "w")
    _need(k_I, torch.bfloat16, None, "k_I")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(idx, torch.int32, (T, topk), "idx")
    _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_indexer_topk(_ptr(q_I), _ptr(w), _ptr(k_I), k_I.shape[0], _ptr(kv_start), _ptr(n_vis), T,
                                  int(max_n_vis), topk, _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)))


def dsa_topk(scores, n_vis, topk, idx, stream=None):
    import torch
    T = n_vis.shape[0]
    _need(scores, torch.float32, None, "scores")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(idx, torch.int32, (T, topk), "idx")
    _check(lib().dsa_topk(_ptr(scores), scores.shape[1], _ptr(n_vis), T, topk, _ptr(idx), _stream(stream)))


def dsa_sparse_mla_attn(q, kv, kv_start, idx, scale, o_lat, lse=None, ws=None, stream=None):
    import torch
    T, topk = idx.shape
    _need(q, torch.bfloat16, (T, HEADS, ROW), "q")
    _need(kv, torch.bfloat16, None, "kv")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(idx, torch.int32, (T, topk), "idx")
    _need(o_lat, torch.float32, (T, HEADS, LATENT), "o_lat")
    if lse is not None:
        _need(lse, torch.float32, (T, HEADS), "lse")
    if ws is not None:
        _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_sparse_mla_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(kv_start), _ptr(idx), T, topk,
                                     float(scale), _ptr(o_lat), _ptr(lse), _ptr(ws), 0 if ws is None else ws.numel(),
                                     _stream(stream)))


def dsa_dense_sparse_attn(q, kv, kv_start, n_vis, idx, window, gate, scale, o_lat, lse_dense=None, lse_sparse=None,
                          ws=None, stream=None):
    import torch
    T, topk = idx.shape
    _need(q, torch.bfloat16, (T, HEADS, ROW), "q")
    _need(kv, torch.bfloat16, None, "kv")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(idx, torch.int32, (T, topk), "idx")
    _need(gate, torch.float32, (T, HEADS), "gate")
    _need(o_lat, torch.float32, (T, HEADS, LATENT), "o_lat")
    for t, nm in ((lse_dense, "lse_dense"), (lse_sparse, "lse_sparse")):
        if t is not None:
            _need(t, torch.float32, (T, HEADS), nm)
    if ws is not None:
        _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_dense_sparse_attn(_ptr(q), _ptr(kv), kv.shape[0], _ptr(kv_start), _ptr(n_vis), _ptr(idx), T, topk,
                                       int(window), _ptr(gate), float(scale), _ptr(o_lat), _ptr(lse_dense),
                                       _ptr(lse_sparse), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))


def dsa_forward(q_I, w, k_I, q, kv, kv_start, n_vis, max_n_vis, topk, scale, o_lat, lse, idx_out, ws, stream=None):
    import torch
    T = n_vis.shape[0]
    _need(q_I, torch.bfloat16, (T, INDEX_HEADS, INDEX_DIM), "q_I")
    _need(w, torch.bfloat16, (T, INDEX_HEADS), "w")
    _need(k_I, torch.bfloat16, None, "k_I")
    _need(q, torch.bfloat16, (T, HEADS, ROW), "q")
    _need(kv, torch.bfloat16, None, "kv")
    if k_I.shape[0] != kv.shape[0]:
        raise ValueError("k_I and kv must have the same number of cache rows")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(o_lat, torch.float32, (T, HEADS, LATENT), "o_lat")
    if lse is not None:
        _need(lse, torch.float32, (T, HEADS), "lse")
    if idx_out is not None:
        _need(idx_out, torch.int32, (T, topk), "idx_out")
    _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_forward(_ptr(q_I), _ptr(w), _ptr(k_I), _ptr(q), _ptr(kv), kv.shape[0], _ptr(kv_start),
                             _ptr(n_vis), T, int(max_n_vis), topk, float(scale), _ptr(o_lat), _ptr(lse),
                             _ptr(idx_out), _ptr(ws), ws.numel(), _stream(stream)))


def dsa_block_sparse_attn(q_I, w, k_I, q, kv, kv_start, n_vis, max_n_vis, gates, scale, o_lat, lse, blocks_out, ws,
                          stream=None):
    """Block-level variant: local / anchor / top-16-block branches fused with
    gates [T, 64, 3]; lse [3, T, 64] and blocks_out [T, 16] may be None."""
    import torch
    T = n_vis.shape[0]
    for t_, nm in ((q_I, "q_I"), (w, "w"), (k_I, "k_I"), (q, "q"), (kv, "kv")):
        _need(t_, torch.bfloat16, None, nm)
    _need(q_I, torch.bfloat16, (T, INDEX_HEADS, INDEX_DIM), "q_I")
    _need(q, torch.bfloat16, (T, HEADS, ROW), "q")
    _need(kv, torch.bfloat16, (kv.shape[0], ROW), "kv")
    _need(k_I, torch.bfloat16, (kv.shape[0], INDEX_DIM), "k_I")
    _need(kv_start, torch.int64, (T,), "kv_start")
    _need(n_vis, torch.int32, (T,), "n_vis")
    _need(gates, torch.float32, (T, HEADS, 3), "gates")
    _need(o_lat, torch.float32, (T, HEADS, LATENT), "o_lat")
    if lse is not None:
        _need(lse, torch.float32, (3, T, HEADS), "lse")
    if blocks_out is not None:
        _need(blocks_out, torch.int32, (T, BLOCK_TOPK), "blocks_out")
    _need(ws, torch.uint8, None, "ws")
    _check(lib().dsa_block_sparse_attn(_ptr(q_I), _ptr(w), _ptr(k_I), _ptr(q), _ptr(kv), kv.shape[0], _ptr(kv_start),
                                       _ptr(n_vis), T, int(max_n_vis), _ptr(gates), float(scale), _ptr(o_lat),
                                       _ptr(lse), _ptr(blocks_out), _ptr(ws), ws.numel(), _stream(stream)))


def dsa_sync_status(stream=None):
    _check(lib().dsa_sync_status(_stream(stream)))


def dsa_set_wait_limit_ns(ns: int):
    """Limit of every bounded device wait, in ns (0: the default)."""
    lib().dsa_set_wait_limit_ns(int(ns))


def dsa_check_wait_timeout(stream=None):
    """Enqueue the hang-protection probe (a wait nothing completes); the next
    dsa_sync_status reports DSA_ERR_TIMEOUT."""
    _check(lib().dsa_check_wait_timeout(_stream(stream)))


def workspace(op, T, max_n_vis, topk, device=None):
    """Allocate a workspace tensor (torch owns the memory; 256-byte aligned)."""
    import torch
    n = max(dsa_workspace_size(op, T, max_n_vis, topk), 256)
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")
