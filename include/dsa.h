/*
 * dsa.h — C ABI of libdsa, the B200 (sm_100a) DSA sparse-attention step:
 * lightning indexer -> per-row top-k -> sparse MLA attention in latent form.
 *
 * What the step computes (pages on the method; page title and section):
 *  - "2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2: a lightweight
 *    indexer scores every query against all of its history and is used only
 *    to rank; a top-k selector keeps index_topk = 2048 positions; real MLA
 *    attention runs over those positions only.
 *  - same page, section 2.1 (config table): index_n_heads 32,
 *    index_head_dim 128, num_attention_heads 64, kv_lora_rank 512,
 *    qk_rope_head_dim 64, qk_head_dim 256, index_topk 2048.
 *  - "From a trillion dot products to two thousand: how DSA breaks N^2", section "DSA full flow": indexer over all
 *    history -> top-2048 -> softmax over the 2048 and the value mix; the KV
 *    cache keeps unselected positions for other queries.
 *  The score and attention formulas (stated on each function) are the
 *  problem statement's; the pages print none.
 *
 * Conventions shared by every entry point
 *  - Every tensor pointer is a caller-owned DEVICE pointer.  The library never
 *    allocates or frees device memory; scratch comes from the caller's `ws`.
 *  - bf16 tensors are passed as their 16-bit patterns (dsa_bf16).
 *  - Each call enqueues work on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns without synchronising.
 *  - Returns DSA_OK or an error code.  Host-side checks (null pointers,
 *    alignment, sizes) fail before anything is enqueued.  Per-row problems
 *    that only the device can see (n_vis or kv_start out of range, an index
 *    outside the cache) make the kernels skip that row and raise a bit in a
 *    device status word; a bounded device wait that expires does the same.
 *    dsa_sync_status() synchronises the stream and reports and clears those
 *    bits.  dsa_last_error_string() describes the last failure of the
 *    calling thread.
 *  - Rows: query row i reads cache rows kv_start[i] .. kv_start[i]+n_vis[i]-1
 *    of a flat cache of `cache_rows` rows.  The query is at position
 *    n_vis[i]-1 of its sequence and sees itself (causal: s <= t, n_vis = t+1).
 *    Positions and indices are relative to kv_start[i].
 *  - The kernels are built for sm_100a only; other devices get
 *    DSA_ERR_UNSUPPORTED.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

#define DSA_INDEX_HEADS 32  /* index_n_heads */
#define DSA_INDEX_DIM 128   /* index_head_dim */
#define DSA_HEADS 64        /* num_attention_heads */
#define DSA_LATENT 512      /* kv_lora_rank: width of c_kv and of o_lat */
#define DSA_ROPE 64         /* qk_rope_head_dim */
#define DSA_ROW 576         /* DSA_LATENT + DSA_ROPE: one latent-cache row / one latent query */
#define DSA_MAX_TOPK 2048   /* index_topk */

typedef uint16_t dsa_bf16;             /* bf16 bit pattern */
typedef struct CUstream_st* dsa_stream_t; /* same type as cudaStream_t */

enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* null / misaligned pointer, bad size (host check) */
  DSA_ERR_WORKSPACE = 2,   /* ws smaller than dsa_workspace_size() */
  DSA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  DSA_ERR_TIMEOUT = 4,     /* a bounded device wait expired (from dsa_sync_status) */
  DSA_ERR_UNSUPPORTED = 5, /* current device is not sm_100 */
  DSA_ERR_BAD_ROW = 6      /* a row had n_vis/kv_start/index out of range and was skipped (from dsa_sync_status) */
};

enum dsa_op {
  DSA_OP_INDEXER = 0,
  DSA_OP_TOPK = 1,
  DSA_OP_SPARSE_MLA = 2,
  DSA_OP_FORWARD = 3,
  DSA_OP_INDEXER_TOPK = 4,
  DSA_OP_DENSE_SPARSE = 5,
  DSA_OP_BLOCK_SPARSE = 6
};

/*
 * Bytes of device workspace `op` needs for T query rows, n_vis <= max_n_vis
 * and the given topk.  Pure host function; 0 means no workspace is needed.
 */
DSA_API size_t dsa_workspace_size(int op, int T, int64_t max_n_vis, int topk);

/*
 * Lightning-indexer scores ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2;
 * "From a trillion dot products to two thousand: how DSA breaks N^2", section "how is the coarse screen fast? low
 * dimensions"):
 *     scores[i, s] = sum_{h<32} w[i,h] * (q_I[i,h,:] . k_I[kv_start[i]+s, :])
 * for 0 <= s < n_vis[i], computed from bf16 inputs with fp32 accumulation on
 * the tensor cores.  Columns s >= n_vis[i] of the row are not written.
 *
 *  q_I     [T,32,128] bf16, row-major, 16-byte aligned
 *  w       [T,32]     bf16, 16-byte aligned
 *  k_I     [cache_rows,128] bf16 (256 B per row), 16-byte aligned
 *  kv_start[T] int64, n_vis[T] int32 (device); need 1 <= n_vis[i] <= score_ld
 *          and 0 <= kv_start[i], kv_start[i]+n_vis[i] <= cache_rows
 *  scores  [T,score_ld] fp32, 16-byte aligned, score_ld % 4 == 0
 *  ws      >= dsa_workspace_size(DSA_OP_INDEXER, T, score_ld, 0) bytes, 256-byte aligned
 */
DSA_API int dsa_indexer_scores(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                       const int64_t* kv_start, const int32_t* n_vis, int T, float* scores, int64_t score_ld,
                       void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Top-k selector ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2: keep the
 * index_topk highest-scoring positions; "From a trillion dot products to two thousand: how DSA breaks N^2",
 * index_topk: 2048).  For row i keeps K = min(topk, n_vis[i]) positions of
 * scores[i, 0:n_vis[i]] under the total order (score descending, position
 * ascending: ties go to the lower position; -0.0 equals +0.0), writes them in
 * ascending position order to idx[i, 0:K] and fills idx[i, K:topk] with -1.
 * Exact: the kept set is the unique top-K of that order.
 *
 *  scores  [T,score_ld] fp32 (16-byte aligned, score_ld % 4 == 0); no NaN
 *  n_vis   [T] int32 (device), 1 <= n_vis[i] <= score_ld
 *  idx     [T,topk] int32, 1 <= topk <= 2048
 */
DSA_API int dsa_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk, int32_t* idx,
             dsa_stream_t stream);

/*
 * Sparse MLA attention in latent (absorbed) form over the selected rows
 * ("From a trillion dot products to two thousand: how DSA breaks N^2", "DSA full flow": full Q.K, softmax and the
 * value mix over the selected 2048 only; config table: qk_head_dim 256 so the
 * softmax scale is 1/sqrt(256)).  For row i, head h and the valid entries
 * s_j = idx[i,j] >= 0:
 *     S[h,j]   = scale * (q[i,h,0:512] . kv[r_j,0:512] + q[i,h,512:576] . kv[r_j,512:576]),
 *                r_j = kv_start[i] + s_j
 *     o_lat[i,h,:] = sum_j softmax_j(S[h,:]) * kv[r_j, 0:512]
 *     lse[i,h]     = log sum_j exp(S[h,j])           (natural log)
 * bf16 inputs, fp32 tensor-core accumulation and fp32 softmax.  A row whose
 * idx holds no valid entry gets o_lat = 0 and lse = -inf.
 *
 *  q       [T,64,576] bf16 (q_lat || q_rope), 16-byte aligned
 *  kv      [cache_rows,576] bf16 (c_kv || k_rope, 1152 B per row), 16-byte aligned
 *  kv_start[T] int64 (device)
 *  idx     [T,topk] int32: positions relative to kv_start, -1 = empty slot;
 *          entries with kv_start+idx >= cache_rows are skipped (status bit)
 *  o_lat   [T,64,512] fp32, 16-byte aligned; lse [T,64] fp32 or NULL
 *  ws      dsa_workspace_size(DSA_OP_SPARSE_MLA, T, 0, topk) bytes, 256-byte
 *          aligned, or NULL.  With few rows the selected positions of a row are
 *          split over several CTAs whose fp32 partial results go to ws and are
 *          merged by a second kernel; a NULL or smaller ws only reduces that
 *          split (down to one CTA per row), never the result.
 */
DSA_API int dsa_sparse_mla_attn(const dsa_bf16* q, const dsa_bf16* kv, int64_t cache_rows, const int64_t* kv_start,
                        const int32_t* idx, int T, int topk, float scale, float* o_lat, float* lse, void* ws,
                        size_t ws_bytes, dsa_stream_t stream);

/*
 * Dense + sparse attention, the two branches of a DSA layer fused ("GLM-5.2's
 * DSA architecture: how dense and sparse attention split the work", section
 * "DSA's core design: dense and sparse side by side": local dense attention over
 * a sliding window next to the current token, global sparse attention over the
 * selected top-k positions, outputs fused inside the layer with learned
 * weights).  For row i with n = n_vis[i], the attention of dsa_sparse_mla_attn
 * is taken twice:
 *     o_sparse over idx[i, 0:topk]
 *     o_dense  over the window positions n - window .. n - 1 (those >= 0)
 *     o_lat[i,h,:] = gate[i,h] * o_dense[i,h,:] + (1 - gate[i,h]) * o_sparse[i,h,:]
 * The pages give neither the window length nor the fusion formula: the window
 * is the caller's, and the learned fusion is read as a per-(row, head) weight
 * gate in [0, 1] supplied by the caller.
 *
 *  q, kv, kv_start, idx, scale, o_lat   as for dsa_sparse_mla_attn
 *  n_vis       [T] int32 (device), n_vis[i] >= 1 (rows with n_vis < 1: status bit, -1 window)
 *  window      1 <= window <= 2048
 *  gate        [T,64] fp32 (device)
 *  lse_dense, lse_sparse  [T,64] fp32 or NULL: each branch's log-sum-exp
 *  ws          >= dsa_workspace_size(DSA_OP_DENSE_SPARSE, T, 0, 0) bytes, 256-byte aligned
 */
DSA_API int dsa_dense_sparse_attn(const dsa_bf16* q, const dsa_bf16* kv, int64_t cache_rows,
                                  const int64_t* kv_start, const int32_t* n_vis, const int32_t* idx, int T, int topk,
                                  int window, const float* gate, float scale, float* o_lat, float* lse_dense,
                                  float* lse_sparse, void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * Block-level variant ("GLM-5: 744B parameters, 202K long context", section 2,
 * "Decoupled Sparse Attention"): the context is cut into 128-token blocks and
 * three branches attend, each over its own positions, fused with weights:
 *  - local:   the query's block and its neighbours (3 x 128 = 384 positions; the
 *             later neighbour is in the future): positions max(0, 128 (qb - 1)) .. t,
 *             qb = t / 128 the query's block, t = n_vis[i] - 1;
 *  - anchor:  one block in every 16: the visible positions of blocks 0, 16, 32, ... <= qb;
 *  - dynamic: the query's 16 most relevant blocks.  The page does not say how a
 *             block is scored; here its score is the largest lightning-indexer
 *             score (dsa_indexer_scores) among its visible positions, and the 16
 *             best blocks are kept under (score descending, block ascending).
 * Each branch is the attention of dsa_sparse_mla_attn over its positions; the
 * page's fusion weights are learned and here come from the caller:
 *     o_lat[i,h,:] = gates[i,h,0] o_local + gates[i,h,1] o_anchor + gates[i,h,2] o_dynamic
 *
 *  q_I, w, k_I, q, kv, cache_rows, kv_start, n_vis, scale   as for dsa_forward
 *  max_n_vis   host-side bound of n_vis (rows above it: status bit, empty branches)
 *  gates       [T,64,3] fp32 (device)
 *  o_lat       [T,64,512] fp32
 *  lse         [3,T,64] fp32 (each branch's log-sum-exp: local, anchor, dynamic) or NULL
 *  blocks_out  [T,16] int32: the dynamic branch's blocks, ascending, -1 padded; or NULL
 *  ws          >= dsa_workspace_size(DSA_OP_BLOCK_SPARSE, T, max_n_vis, 0) bytes, 256-byte
 *              aligned; it holds the T x max_n_vis score matrix (4 bytes per entry)
 */
DSA_API int dsa_block_sparse_attn(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, const dsa_bf16* q,
                                  const dsa_bf16* kv, int64_t cache_rows, const int64_t* kv_start,
                                  const int32_t* n_vis, int T, int64_t max_n_vis, const float* gates, float scale,
                                  float* o_lat, float* lse, int32_t* blocks_out, void* ws, size_t ws_bytes,
                                  dsa_stream_t stream);

/*
 * Indexer and top-k fused, without a score matrix ("2026 LLM architecture
 * overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2: score every
 * history position, keep index_topk of them).  Selects exactly what
 * dsa_indexer_scores followed by dsa_topk selects, but each query's scores
 * are filtered on the fly into a candidate buffer (kept in ws) that is cut
 * back to the current top-k whenever it fills, so no T x n_vis matrix is
 * written.  Rows of equal kv_start are processed together (up to 8), each
 * group by one CTA over its whole context.
 *
 *  arguments as dsa_indexer_scores / dsa_topk; max_n_vis bounds n_vis
 *  idx   [T,topk] int32: ascending positions, -1 padded (rows with invalid
 *        n_vis / kv_start get all -1 and a status bit)
 *  ws    >= dsa_workspace_size(DSA_OP_INDEXER_TOPK, T, max_n_vis, topk) bytes, 256-byte aligned
 */
DSA_API int dsa_indexer_topk(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                             const int64_t* kv_start, const int32_t* n_vis, int T, int64_t max_n_vis, int topk,
                             int32_t* idx, void* ws, size_t ws_bytes, dsa_stream_t stream);

/*
 * The whole step: indexer -> top-k -> sparse MLA, enqueued on one stream.
 * Arguments as above; k_I and kv share the row numbering (cache_rows rows).
 * max_n_vis is a host-side upper bound of n_vis (rows above it are skipped
 * with a status bit).  idx_out [T,topk] receives the selected positions when
 * not NULL.  The score matrix is materialised in `ws` when it is small
 * (T * max_n_vis * 4 bytes within the workspace rule of dsa_workspace_size);
 * otherwise scores are streamed into the selector and never stored.
 */
DSA_API int dsa_forward(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, const dsa_bf16* q, const dsa_bf16* kv,
                int64_t cache_rows, const int64_t* kv_start, const int32_t* n_vis, int T, int64_t max_n_vis, int topk,
                float scale, float* o_lat, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes,
                dsa_stream_t stream);

/*
 * dsa_indexer_scores without a workspace argument: the same scores, for
 * callers that cannot allocate device memory.  There is no counterpart on
 * the pages; this is a library-interface addition.
 *
 * Who needs it: code that runs inside a host framework which owns every
 * byte of device memory and allows no allocation once it has started (a
 * serving engine with a memory pool planned at start-up, a plug-in whose
 * host interface hands it tensors but no allocator).  For such callers
 * cudaMalloc is either unavailable or would synchronise the device in the
 * middle of a step.
 *
 * Scratch: the per-call query-tile plan lives in a fixed array in the
 * library's own device memory (DSA_NOALLOC_MAX_ROWS rows, about 256 KB),
 * which every GPU that loads the library holds until the process exits.
 * T above DSA_NOALLOC_MAX_ROWS is rejected with DSA_ERR_INVALID_ARG.
 * The first call on a device looks up that array's device address (with
 * that device current); make that first call before any stream capture.
 * All calls share the one array and each call overwrites what the previous
 * one left there, so calls whose execution overlaps on the GPU (other
 * streams, other host threads) race and must be serialised by the caller.
 * Arguments and errors otherwise as dsa_indexer_scores.
 */
#define DSA_NOALLOC_MAX_ROWS 8192
DSA_API int dsa_indexer_scores_noalloc(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I,
                                       int64_t cache_rows, const int64_t* kv_start, const int32_t* n_vis, int T,
                                       float* scores, int64_t score_ld, dsa_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the device status word of the
 * current device.  Returns DSA_OK, DSA_ERR_TIMEOUT, DSA_ERR_BAD_ROW or
 * DSA_ERR_CUDA (a sticky CUDA error).
 *
 * The status word is one per device, not one per call or per stream: every
 * kernel of the library on that device raises its bits in the same word.  A
 * call on another stream that is still running may raise a bit after this
 * one synchronised, and the first caller to read the word reports and clears
 * the bits of every call that ran before it, whatever its stream.  Callers
 * that drive several streams on one device should read the status at a point
 * where the calls they want to attribute it to are the only ones that ran.
 */
DSA_API int dsa_sync_status(dsa_stream_t stream);

/*
 * Limit, in nanoseconds, of every bounded device wait the library's kernels
 * make (TMA, tensor-core and producer/consumer hand-offs).  A wait that runs
 * past it gives up: its CTA stops its work, lets every copy and tensor-core
 * operation it started finish, releases its resources and exits, and the
 * timeout bit reported by dsa_sync_status as DSA_ERR_TIMEOUT is raised; the
 * outputs of that call are then undefined, the CUDA context stays usable.
 * 0 restores the default (environment variable DSA_WAIT_LIMIT_NS, else
 * 1.5 s).  Takes effect for launches after the call; process-wide.
 */
DSA_API void dsa_set_wait_limit_ns(unsigned long long ns);

/*
 * Diagnostic of the hang protection: enqueues one CTA on `stream` that waits,
 * under the current wait limit, on a barrier that nothing ever completes.
 * The wait must give up; a following dsa_sync_status(stream) then returns
 * DSA_ERR_TIMEOUT (and clears the bit).  With the default limit the probe
 * takes 1.5 s; set a short limit first with dsa_set_wait_limit_ns.
 */
DSA_API int dsa_check_wait_timeout(dsa_stream_t stream);

/* Message for the calling thread's last failure ("" if none). Never NULL. */
DSA_API const char* dsa_last_error_string(void);

/* ABI version of this header: 1. */
DSA_API int dsa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
