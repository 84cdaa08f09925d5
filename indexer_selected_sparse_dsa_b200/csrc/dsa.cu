// libdsa: the C ABI declared in include/dsa.h, and the only translation unit
// of the library (the kernels are included below so they share one device
// status word without relocatable device code).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <string>

#include "dsa.h"
#include "internal.h"
#include "ptx.cuh"

#include "block_sparse.cuh"
#include "dense_sparse.cuh"
#include "indexer.cuh"
#include "sparse_mla.cuh"
#include "topk.cuh"
#include "decode_fused.cuh"

// Scratch of dsa_indexer_scores_noalloc: the query-tile plan for up to
// DSA_NOALLOC_MAX_ROWS rows (about 256 KB).  Every device that loads this
// library holds its own copy until the process exits; all calls of that entry
// point on a device share it.
static constexpr size_t kNoAllocPlanBytes =
    sizeof(dsa::PlanHeader) + sizeof(dsa::PlanTile) * size_t(DSA_NOALLOC_MAX_ROWS);
static __device__ __align__(256) unsigned char g_noalloc_plan[kNoAllocPlanBytes];

namespace {

thread_local std::string t_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(DSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- per-device state
struct DeviceState {
  bool probed = false;
  bool supported = false;
  bool prepared = false;
  bool cooperative = false;
  int sm_count = 0;
  void* noalloc_plan = nullptr;  // device address of g_noalloc_plan on this device
};
constexpr int kMaxDevices = 64;
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

int current_device(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceState& d = g_dev[dev];
  if (!d.probed) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    int coop = 0;
    if ((e = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.supported = (major == 10 && minor == 0);
    d.cooperative = coop != 0;
    d.sm_count = sms;
    d.probed = true;
  }
  if (!d.supported) return fail(DSA_ERR_UNSUPPORTED, "libdsa is built for sm_100a; device %d is not", dev);
  if (!d.prepared) {
    if ((e = dsa::prepare_indexer()) != cudaSuccess) return cuda_fail(e, "indexer smem opt-in");
    if ((e = dsa::prepare_sparse_mla()) != cudaSuccess) return cuda_fail(e, "sparse MLA smem opt-in");
    if ((e = dsa::prepare_topk()) != cudaSuccess) return cuda_fail(e, "top-k smem opt-in");
    if ((e = dsa::prepare_decode_fused()) != cudaSuccess) return cuda_fail(e, "fused decode smem opt-in");
    d.prepared = true;
  }
  *out = &d;
  return DSA_OK;
}

// Limit of every bounded device wait: dsa_set_wait_limit_ns, else the
// environment variable DSA_WAIT_LIMIT_NS, else 1.5 s.  Read at each launch.
std::atomic<unsigned long long> g_wait_limit_override{0};

unsigned long long wait_limit_ns() {
  const unsigned long long o = g_wait_limit_override.load(std::memory_order_relaxed);
  if (o > 0) return o;
  static const unsigned long long v = [] {
    const char* s = std::getenv("DSA_WAIT_LIMIT_NS");
    if (s && *s) {
      unsigned long long x = std::strtoull(s, nullptr, 10);
      if (x > 0) return x;
    }
    return 1500000000ull;  // 1.5 s per wait
  }();
  return v;
}

// One CTA waits on an mbarrier that nothing ever completes, under the current
// wait limit: the wait must give up and raise the timeout bit.
__global__ void wait_probe_kernel(dsa::WaitLimit lim) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = dsa::smem_u32(&bar);
  if (threadIdx.x == 0) {
    dsa::mbar_init(b, 1);
    dsa::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) dsa::mbar_wait(b, 0, lim, nullptr);
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return EncodeTiledFn(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D bf16 row-major [rows, cols] tensor map with a box of [box_rows, 64] and 128-byte swizzle.
int make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", int(r));
  return DSA_OK;
}

// ---------------------------------------------------------------- sizes
int64_t score_ld_for(int64_t max_n_vis) { return (max_n_vis + 3) / 4 * 4; }

size_t ws_indexer(int T) { return align_up(dsa::indexer_plan_bytes(T), 256); }

size_t ws_mla(int T, int topk) { return align_up(dsa::sparse_mla_part_bytes(T, dsa::sparse_mla_ws_splits(T, topk)), 256); }

// dsa_forward streams scores into the selector (never stores them) when the score
// matrix would be larger than this; DSA_FORWARD_MODE=stream|materialize overrides.
constexpr size_t kStreamAboveBytes = size_t(8) << 30;

bool forward_streams(int T, int64_t max_n_vis) {
  if (const char* m = std::getenv("DSA_FORWARD_MODE")) {
    if (!std::strcmp(m, "stream")) return true;
    if (!std::strcmp(m, "materialize")) return false;
  }
  return size_t(T) * size_t(score_ld_for(max_n_vis)) * 4 > kStreamAboveBytes;
}

size_t ws_candidates(int T) { return align_up(size_t(T) * dsa::kStreamCap * 4, 256); }
// streamed selection: candidate keys, candidate positions, the redo list, the candidate counts
size_t ws_redo(int T) { return align_up((size_t(T) + 1) * 4, 256); }
size_t ws_select(int T) { return 2 * ws_candidates(T) + ws_redo(T) + align_up(size_t(T) * 4, 256); }

dsa::StreamOut stream_out_at(uint8_t* sel, int T, int32_t* idx, int topk) {
  dsa::StreamOut so{};
  so.cand_key = reinterpret_cast<uint32_t*>(sel);
  so.cand_pos = reinterpret_cast<int32_t*>(sel + ws_candidates(T));
  so.idx = idx;
  so.topk = topk;
  so.cap = dsa::kStreamCap;
  so.redo = reinterpret_cast<int*>(sel + 2 * ws_candidates(T));
  so.cnt_out = reinterpret_cast<int*>(sel + 2 * ws_candidates(T) + ws_redo(T));
  so.sample_units = dsa::kSampleUnits;
  so.sample_mode = 1;
  // DSA_STREAM_SAMPLE=0: no seeding; =2: seed at the sample maximum (tests of the redo sweep)
  if (const char* m = std::getenv("DSA_STREAM_SAMPLE")) {
    if (m[0] == '0') so.sample_units = 0;
    if (m[0] == '2') so.sample_mode = 2;
  }
  return so;
}

// The fused decode step (small batches): handoff counters and histograms, the
// kept-position bitmaps and the candidate lists, after dsa_forward's own buffers.
bool fused_fits(int T, int64_t max_n_vis) {
  return T >= 1 && T <= dsa::kDecodeMaxRows && score_ld_for(max_n_vis) <= dsa::kDecodeMaxN;
}
struct FusedLayout {
  size_t off_sync, off_cand, total;
};
FusedLayout fused_layout(size_t base, int T, int64_t max_n_vis) {
  const int64_t ld = score_ld_for(max_n_vis);
  FusedLayout L{};
  L.off_sync = base;
  L.off_cand = L.off_sync + align_up(dsa::decode_fused_sync_bytes(), 256);
  L.total = L.off_cand + align_up(size_t(T) * size_t(ld) * 8, 256);
  return L;
}

size_t ws_forward_base(int T, int64_t max_n_vis, int topk) {
  const size_t sel = forward_streams(T, max_n_vis) ? ws_select(T)
                                                   : align_up(size_t(T) * size_t(score_ld_for(max_n_vis)) * 4, 256);
  return ws_indexer(T) + sel + align_up(size_t(T) * size_t(topk) * 4, 256) + ws_mla(T, topk);
}

size_t ws_forward(int T, int64_t max_n_vis, int topk) {
  const size_t base = ws_forward_base(T, max_n_vis, topk);
  return fused_fits(T, max_n_vis) ? fused_layout(base, T, max_n_vis).total : base;
}

// DSA_DECODE_FUSED=1 runs small batches as the one-launch step (decode_fused.cuh);
// by default they take the separate kernels, which are faster today.
bool fused_enabled() {
  const char* s = std::getenv("DSA_DECODE_FUSED");
  return s && s[0] == '1';
}

// dense + sparse: window index rows (up to DSA_MAX_TOPK wide), the dense branch's
// output, then the attention partials
size_t ws_dense_sparse(int T) {
  return align_up(size_t(T) * DSA_MAX_TOPK * 4, 256) + align_up(size_t(T) * DSA_HEADS * DSA_LATENT * 4, 256) +
         ws_mla(T, DSA_MAX_TOPK);
}

// block-level variant: the indexer plan, the score matrix, block scores and counts,
// the dynamic blocks, the three index lists, the local and anchor outputs, the
// attention partials
struct BlockLayout {
  int64_t ld, bld;
  int wa;
  size_t off_scores, off_bscore, off_nblocks, off_blocks, off_loc, off_anc, off_dyn, off_oloc, off_oanc, off_part,
      part_bytes, total;
};
BlockLayout block_layout(int T, int64_t max_n_vis) {
  BlockLayout L{};
  L.ld = score_ld_for(max_n_vis);
  const int64_t nb = (max_n_vis + dsa::kBlockTokens - 1) / dsa::kBlockTokens;
  L.bld = (nb + 3) / 4 * 4;
  L.wa = int((nb + dsa::kAnchorEvery - 1) / dsa::kAnchorEvery) * dsa::kBlockTokens;
  const size_t t = size_t(T);
  size_t o = ws_indexer(T);
  L.off_scores = o;
  o += align_up(t * size_t(L.ld) * 4, 256);
  L.off_bscore = o;
  o += align_up(t * size_t(L.bld) * 4, 256);
  L.off_nblocks = o;
  o += align_up(t * 4, 256);
  L.off_blocks = o;
  o += align_up(t * dsa::kBlockTopk * 4, 256);
  L.off_loc = o;
  o += align_up(t * dsa::kLocalWidth * 4, 256);
  L.off_anc = o;
  o += align_up(t * size_t(L.wa) * 4, 256);
  L.off_dyn = o;
  o += align_up(t * dsa::kDynWidth * 4, 256);
  L.off_oloc = o;
  o += align_up(t * DSA_HEADS * DSA_LATENT * 4, 256);
  L.off_oanc = o;
  o += align_up(t * DSA_HEADS * DSA_LATENT * 4, 256);
  L.off_part = o;
  L.part_bytes = ws_mla(T, L.wa > dsa::kDynWidth ? L.wa : dsa::kDynWidth);
  L.total = o + L.part_bytes;
  return L;
}

int pick_qmax(int T) {
  const char* s = std::getenv("DSA_INDEXER_QMAX");
  if (s && *s) {
    int v = std::atoi(s);
    if (v == 1 || v == 4 || v == 8) return v;
  }
  return T >= 5 ? 8 : (T >= 2 ? 4 : 1);
}

int check_common_rows(int T, int64_t cache_rows, const void* kv_start) {
  if (T < 0) return fail(DSA_ERR_INVALID_ARG, "T must be >= 0 (got %d)", T);
  if (cache_rows < 1 || cache_rows > INT32_MAX)
    return fail(DSA_ERR_INVALID_ARG, "cache_rows must lie in [1, 2^31-1] (got %lld)", (long long)cache_rows);
  if (T > 0 && !kv_start) return fail(DSA_ERR_INVALID_ARG, "kv_start is NULL");
  if (!aligned(kv_start, 8)) return fail(DSA_ERR_INVALID_ARG, "kv_start must be 8-byte aligned");
  return DSA_OK;
}

int run_sparse_mla(const dsa::MlaLaunch& p) {
  if (int64_t(p.T) * DSA_HEADS > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "T too large");
  CUtensorMap tq;
  int rc = make_tmap_bf16(&tq, p.q, DSA_ROW, uint64_t(p.T) * DSA_HEADS, 64);
  if (rc) return rc;
  cudaError_t e = dsa::launch_sparse_mla(p, tq);
  if (e != cudaSuccess) return cuda_fail(e, "sparse MLA launch");
  return DSA_OK;
}

int run_indexer(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                const int64_t* kv_start, const int32_t* n_vis, int T, float* scores, int64_t score_ld, void* plan,
                dsa_stream_t stream, int sm_count, const dsa::StreamOut* stream_out = nullptr) {
  int qmax = stream_out ? 8 : pick_qmax(T);
  CUtensorMap tk, tq;
  int rc = make_tmap_bf16(&tk, k_I, DSA_INDEX_DIM, uint64_t(cache_rows), 128);
  if (rc) return rc;
  rc = make_tmap_bf16(&tq, q_I, DSA_INDEX_DIM, uint64_t(T) * DSA_INDEX_HEADS, 32);
  if (rc) return rc;
  dsa::IndexerLaunch p{};
  p.q_I = q_I;
  p.w = w;
  p.k_I = k_I;
  p.cache_rows = cache_rows;
  p.kv_start = kv_start;
  p.n_vis = n_vis;
  p.T = T;
  p.scores = scores;
  p.score_ld = score_ld;
  p.plan = plan;
  p.qmax = qmax;
  // Wave sweep when many query tiles share a key set larger than a good part of L2:
  // all CTAs then walk the keys in step and each key tile leaves HBM about once per wave.
  const int n_tiles_min = (T + qmax - 1) / qmax;
  p.sweep = (n_tiles_min >= sm_count && score_ld * 256 > (64ll << 20)) ? dsa::kSweepWave : dsa::kSweepSplit;
  if (const char* sw = std::getenv("DSA_INDEXER_SWEEP")) {
    if (!std::strcmp(sw, "wave")) p.sweep = dsa::kSweepWave;
    if (!std::strcmp(sw, "split")) p.sweep = dsa::kSweepSplit;
  }
  p.streaming = stream_out != nullptr;
  if (stream_out) {
    p.stream_out = *stream_out;
    p.sweep = dsa::kSweepWave;  // a CTA owns each query tile's whole sweep and its selection state
  }
  p.grid = sm_count;
  p.wait_ns = wait_limit_ns();
  p.stream = stream;
  cudaError_t e = dsa::launch_indexer(p, tk, tq);
  if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
  if (stream_out && (e = dsa::launch_stream_select(*stream_out, n_vis, T, stream)) != cudaSuccess)
    return cuda_fail(e, "streamed top-k launch");
  return DSA_OK;
}

}  // namespace

namespace dsa {
bool pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("DSA_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}
}  // namespace dsa

extern "C" {

int dsa_abi_version(void) { return 1; }

const char* dsa_last_error_string(void) { return t_err.c_str(); }

size_t dsa_workspace_size(int op, int T, int64_t max_n_vis, int topk) {
  if (T < 0) T = 0;
  if (max_n_vis < 0) max_n_vis = 0;
  if (topk < 0) topk = 0;
  switch (op) {
    case DSA_OP_INDEXER: return ws_indexer(T);
    case DSA_OP_TOPK: return 0;
    case DSA_OP_SPARSE_MLA: return ws_mla(T, topk);
    case DSA_OP_FORWARD: return ws_forward(T, max_n_vis, topk);
    case DSA_OP_INDEXER_TOPK: return ws_indexer(T) + ws_select(T);
    case DSA_OP_DENSE_SPARSE: return ws_dense_sparse(T);
    case DSA_OP_BLOCK_SPARSE: return max_n_vis > 0 ? block_layout(T, max_n_vis).total : 0;
    default: return 0;
  }
}

int dsa_indexer_scores(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                       const int64_t* kv_start, const int32_t* n_vis, int T, float* scores, int64_t score_ld,
                       void* ws, size_t ws_bytes, dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (T == 0) return DSA_OK;
  if (!q_I || !w || !k_I || !n_vis || !scores || !ws)
    return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_I, 16) || !aligned(w, 16) || !aligned(k_I, 16) || !aligned(scores, 16) || !aligned(n_vis, 4))
    return fail(DSA_ERR_INVALID_ARG, "q_I, w, k_I, scores must be 16-byte aligned and n_vis 4-byte aligned");
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (score_ld < 4 || score_ld % 4 != 0) return fail(DSA_ERR_INVALID_ARG, "score_ld must be a positive multiple of 4");
  if (int64_t(T) * DSA_INDEX_HEADS > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "T too large");
  if (ws_bytes < ws_indexer(T))
    return fail(DSA_ERR_WORKSPACE, "workspace %zu < required %zu bytes", ws_bytes, ws_indexer(T));
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  return run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, scores, score_ld, ws, stream, dev->sm_count);
}

int dsa_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk, int32_t* idx,
             dsa_stream_t stream) {
  t_err.clear();
  if (T < 0) return fail(DSA_ERR_INVALID_ARG, "T must be >= 0");
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_INVALID_ARG, "topk must lie in [1, %d]", DSA_MAX_TOPK);
  if (T == 0) return DSA_OK;
  if (!scores || !n_vis || !idx) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(scores, 16) || !aligned(n_vis, 4) || !aligned(idx, 4))
    return fail(DSA_ERR_INVALID_ARG, "scores must be 16-byte aligned, n_vis and idx 4-byte aligned");
  if (score_ld < 4 || score_ld % 4 != 0) return fail(DSA_ERR_INVALID_ARG, "score_ld must be a positive multiple of 4");
  if (score_ld > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "score_ld too large");
  DeviceState* dev = nullptr;
  int rc = current_device(&dev);
  if (rc) return rc;
  cudaError_t e = dsa::launch_topk(scores, score_ld, n_vis, T, topk, idx, dev->sm_count, stream);
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  return DSA_OK;
}

int dsa_sparse_mla_attn(const dsa_bf16* q, const dsa_bf16* kv, int64_t cache_rows, const int64_t* kv_start,
                        const int32_t* idx, int T, int topk, float scale, float* o_lat, float* lse, void* ws,
                        size_t ws_bytes, dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_INVALID_ARG, "topk must lie in [1, %d]", DSA_MAX_TOPK);
  if (T == 0) return DSA_OK;
  if (!q || !kv || !idx || !o_lat) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(o_lat, 16) || !aligned(idx, 4) || !aligned(lse, 4))
    return fail(DSA_ERR_INVALID_ARG, "q, kv, o_lat must be 16-byte aligned; idx, lse 4-byte aligned");
  if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (ws && !aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  // A workspace smaller than dsa_workspace_size only lowers how many CTAs share a row.
  dsa::MlaLaunch p{q,     kv,  cache_rows, kv_start, idx, T, topk, scale, o_lat, lse, static_cast<float*>(ws),
                   ws ? ws_bytes : 0, dev->sm_count, wait_limit_ns(), stream};
  return run_sparse_mla(p);
}

int dsa_dense_sparse_attn(const dsa_bf16* q, const dsa_bf16* kv, int64_t cache_rows, const int64_t* kv_start,
                          const int32_t* n_vis, const int32_t* idx, int T, int topk, int window, const float* gate,
                          float scale, float* o_lat, float* lse_dense, float* lse_sparse, void* ws, size_t ws_bytes,
                          dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_INVALID_ARG, "topk must lie in [1, %d]", DSA_MAX_TOPK);
  if (window < 1 || window > DSA_MAX_TOPK)
    return fail(DSA_ERR_INVALID_ARG, "window must lie in [1, %d]", DSA_MAX_TOPK);
  if (T == 0) return DSA_OK;
  if (!q || !kv || !n_vis || !idx || !gate || !o_lat || !ws)
    return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(o_lat, 16) || !aligned(n_vis, 4) || !aligned(idx, 4) ||
      !aligned(gate, 4) || !aligned(lse_dense, 4) || !aligned(lse_sparse, 4))
    return fail(DSA_ERR_INVALID_ARG, "q, kv, o_lat must be 16-byte aligned; n_vis, idx, gate, lse 4-byte aligned");
  if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (int64_t(T) * DSA_HEADS > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "T too large");
  const size_t need = ws_dense_sparse(T);
  if (ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu < required %zu bytes", ws_bytes, need);
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* idx_w = reinterpret_cast<int32_t*>(base);
  float* o_dense = reinterpret_cast<float*>(base + align_up(size_t(T) * DSA_MAX_TOPK * 4, 256));
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(o_dense) +
                                         align_up(size_t(T) * DSA_HEADS * DSA_LATENT * 4, 256));
  const size_t part_bytes = ws_mla(T, DSA_MAX_TOPK);
  // sparse branch into o_lat
  dsa::MlaLaunch ps{q,          kv,         cache_rows,   kv_start,      idx,           T,     topk, scale,
                    o_lat,      lse_sparse, part,         part_bytes,    dev->sm_count, wait_limit_ns(), stream};
  if ((rc = run_sparse_mla(ps))) return rc;
  // dense branch over the window, into the workspace
  cudaError_t e = dsa::launch_window_idx(n_vis, T, window, idx_w, stream);
  if (e != cudaSuccess) return cuda_fail(e, "window index launch");
  dsa::MlaLaunch pd{q,          kv,         cache_rows,   kv_start,      idx_w,         T,     window, scale,
                    o_dense,    lse_dense,  part,         part_bytes,    dev->sm_count, wait_limit_ns(), stream};
  if ((rc = run_sparse_mla(pd))) return rc;
  e = dsa::launch_fuse(o_lat, o_dense, gate, T, dev->sm_count, stream);
  if (e != cudaSuccess) return cuda_fail(e, "fusion launch");
  return DSA_OK;
}

int dsa_indexer_topk(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                     const int64_t* kv_start, const int32_t* n_vis, int T, int64_t max_n_vis, int topk, int32_t* idx,
                     void* ws, size_t ws_bytes, dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_INVALID_ARG, "topk must lie in [1, %d]", DSA_MAX_TOPK);
  if (T == 0) return DSA_OK;
  if (max_n_vis < 1 || max_n_vis > cache_rows)
    return fail(DSA_ERR_INVALID_ARG, "max_n_vis must lie in [1, cache_rows]");
  if (!q_I || !w || !k_I || !n_vis || !idx || !ws) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_I, 16) || !aligned(w, 16) || !aligned(k_I, 16) || !aligned(n_vis, 4) || !aligned(idx, 4))
    return fail(DSA_ERR_INVALID_ARG, "q_I, w, k_I must be 16-byte aligned; n_vis, idx 4-byte aligned");
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (int64_t(T) * DSA_INDEX_HEADS > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "T too large");
  const size_t need = ws_indexer(T) + ws_select(T);
  if (ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu < required %zu bytes", ws_bytes, need);
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* sel = base + ws_indexer(T);
  cudaError_t e = cudaMemsetAsync(idx, 0xFF, size_t(T) * size_t(topk) * 4, stream);  // rejected rows stay -1
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(idx)");
  const dsa::StreamOut so = stream_out_at(sel, T, idx, topk);
  return run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, nullptr, score_ld_for(max_n_vis), base, stream,
                     dev->sm_count, &so);
}

int dsa_forward(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, const dsa_bf16* q, const dsa_bf16* kv,
                int64_t cache_rows, const int64_t* kv_start, const int32_t* n_vis, int T, int64_t max_n_vis, int topk,
                float scale, float* o_lat, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes,
                dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (topk < 1 || topk > DSA_MAX_TOPK) return fail(DSA_ERR_INVALID_ARG, "topk must lie in [1, %d]", DSA_MAX_TOPK);
  if (T == 0) return DSA_OK;
  if (max_n_vis < 1 || max_n_vis > cache_rows)
    return fail(DSA_ERR_INVALID_ARG, "max_n_vis must lie in [1, cache_rows]");
  if (!q_I || !w || !k_I || !q || !kv || !n_vis || !o_lat || !ws)
    return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_I, 16) || !aligned(w, 16) || !aligned(k_I, 16) || !aligned(q, 16) || !aligned(kv, 16) ||
      !aligned(o_lat, 16) || !aligned(n_vis, 4) || !aligned(lse, 4) || !aligned(idx_out, 4))
    return fail(DSA_ERR_INVALID_ARG, "tensor pointers misaligned (bf16/o_lat 16 B, n_vis/lse/idx 4 B)");
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "scale must be positive and finite");
  const size_t need = ws_forward(T, max_n_vis, topk);
  if (ws_bytes < need) return fail(DSA_ERR_WORKSPACE, "workspace %zu < required %zu bytes", ws_bytes, need);
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;

  const int64_t ld = score_ld_for(max_n_vis);
  const bool streams = forward_streams(T, max_n_vis);
  uint8_t* base = static_cast<uint8_t*>(ws);
  // Small batches: one cooperative launch when every attention tile and every
  // query's selection gets a CTA of its own.
  if (fused_enabled() && !streams && dev->cooperative && fused_fits(T, max_n_vis) &&
      int64_t(T) * ((std::min<int64_t>(topk, max_n_vis) + 127) / 128) + T <= dev->sm_count) {
    const FusedLayout FL = fused_layout(ws_forward_base(T, max_n_vis, topk), T, max_n_vis);
    uint8_t* sel0 = base + ws_indexer(T);
    const size_t sel_bytes0 = align_up(size_t(T) * size_t(ld) * 4, 256);
    int32_t* idx_ws0 = reinterpret_cast<int32_t*>(sel0 + sel_bytes0);
    float* part0 = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(idx_ws0) +
                                            align_up(size_t(T) * size_t(topk) * 4, 256));
    CUtensorMap tk, tqi, tq;
    if ((rc = make_tmap_bf16(&tk, k_I, DSA_INDEX_DIM, uint64_t(cache_rows), 128))) return rc;
    if ((rc = make_tmap_bf16(&tqi, q_I, DSA_INDEX_DIM, uint64_t(T) * DSA_INDEX_HEADS, 32))) return rc;
    if ((rc = make_tmap_bf16(&tq, q, DSA_ROW, uint64_t(T) * DSA_HEADS, 64))) return rc;
    dsa::DecodeFusedLaunch fp{};
    fp.w = w;
    fp.kv = kv;
    fp.kv_start = kv_start;
    fp.n_vis = n_vis;
    fp.T = T;
    fp.topk = topk;
    fp.cache_rows = cache_rows;
    fp.score_ld = ld;
    fp.scale = scale;
    fp.scores = reinterpret_cast<float*>(sel0);
    fp.cand = base + FL.off_cand;
    fp.sync = reinterpret_cast<uint32_t*>(base + FL.off_sync);
    fp.part = part0;
    fp.o_lat = o_lat;
    fp.lse = lse;
    fp.idx = idx_out ? idx_out : idx_ws0;
    fp.sm_count = dev->sm_count;
    fp.wait_ns = wait_limit_ns();
    fp.stream = stream;
    cudaError_t e = dsa::launch_decode_fused(fp, tk, tqi, tq);
    if (e != cudaSuccess) return cuda_fail(e, "fused decode launch");
    return DSA_OK;
  }
  void* plan = base;
  uint8_t* sel = base + ws_indexer(T);  // score matrix, or the candidate buffers
  const size_t sel_bytes = streams ? ws_select(T) : align_up(size_t(T) * size_t(ld) * 4, 256);
  int32_t* idx_ws = reinterpret_cast<int32_t*>(sel + sel_bytes);
  int32_t* idx = idx_out ? idx_out : idx_ws;
  float* part = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(idx_ws) + align_up(size_t(T) * size_t(topk) * 4, 256));

  cudaError_t e;
  if (streams) {
    // Rows the indexer plan rejects are never visited: they keep -1 everywhere.
    if ((e = cudaMemsetAsync(idx, 0xFF, size_t(T) * size_t(topk) * 4, stream)) != cudaSuccess)
      return cuda_fail(e, "cudaMemsetAsync(idx)");
    const dsa::StreamOut so = stream_out_at(sel, T, idx, topk);
    if ((rc = run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, nullptr, ld, plan, stream, dev->sm_count,
                          &so)))
      return rc;
  } else {
    float* scores = reinterpret_cast<float*>(sel);
    if ((rc = run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, scores, ld, plan, stream, dev->sm_count)))
      return rc;
    e = dsa::launch_topk(scores, ld, n_vis, T, topk, idx, dev->sm_count, stream);
    if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  }
  dsa::MlaLaunch p{q,    kv,  cache_rows,        kv_start,      idx,           T,     topk, scale,
                   o_lat, lse, part,              ws_mla(T, topk), dev->sm_count, wait_limit_ns(), stream};
  return run_sparse_mla(p);
}

int dsa_block_sparse_attn(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, const dsa_bf16* q,
                          const dsa_bf16* kv, int64_t cache_rows, const int64_t* kv_start, const int32_t* n_vis, int T,
                          int64_t max_n_vis, const float* gates, float scale, float* o_lat, float* lse,
                          int32_t* blocks_out, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (T == 0) return DSA_OK;
  if (max_n_vis < 1 || max_n_vis > cache_rows)
    return fail(DSA_ERR_INVALID_ARG, "max_n_vis must lie in [1, cache_rows]");
  if (!q_I || !w || !k_I || !q || !kv || !n_vis || !gates || !o_lat || !ws)
    return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_I, 16) || !aligned(w, 16) || !aligned(k_I, 16) || !aligned(q, 16) || !aligned(kv, 16) ||
      !aligned(o_lat, 16) || !aligned(n_vis, 4) || !aligned(gates, 4) || !aligned(lse, 4) || !aligned(blocks_out, 4))
    return fail(DSA_ERR_INVALID_ARG, "tensor pointers misaligned (bf16/o_lat 16 B, n_vis/gates/lse/blocks 4 B)");
  if (!aligned(ws, 256)) return fail(DSA_ERR_INVALID_ARG, "ws must be 256-byte aligned");
  if (!(scale > 0.f) || !(scale < 1e30f)) return fail(DSA_ERR_INVALID_ARG, "scale must be positive and finite");
  if (int64_t(T) * DSA_HEADS > INT32_MAX) return fail(DSA_ERR_INVALID_ARG, "T too large");
  const BlockLayout L = block_layout(T, max_n_vis);
  if (ws_bytes < L.total) return fail(DSA_ERR_WORKSPACE, "workspace %zu < required %zu bytes", ws_bytes, L.total);
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(base + L.off_scores);
  float* bscore = reinterpret_cast<float*>(base + L.off_bscore);
  int32_t* nblocks = reinterpret_cast<int32_t*>(base + L.off_nblocks);
  int32_t* blocks = blocks_out ? blocks_out : reinterpret_cast<int32_t*>(base + L.off_blocks);
  int32_t* idx_loc = reinterpret_cast<int32_t*>(base + L.off_loc);
  int32_t* idx_anc = reinterpret_cast<int32_t*>(base + L.off_anc);
  int32_t* idx_dyn = reinterpret_cast<int32_t*>(base + L.off_dyn);
  float* o_loc = reinterpret_cast<float*>(base + L.off_oloc);
  float* o_anc = reinterpret_cast<float*>(base + L.off_oanc);
  float* part = reinterpret_cast<float*>(base + L.off_part);
  if ((rc = run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, scores, L.ld, base, stream, dev->sm_count)))
    return rc;
  cudaError_t e = dsa::launch_block_max(scores, L.ld, n_vis, T, int(L.bld), bscore, nblocks, stream);
  if (e != cudaSuccess) return cuda_fail(e, "block score launch");
  // the 16 best blocks of each row: the exact top-k over block scores (ties to the lower block)
  if ((e = dsa::launch_topk(bscore, L.bld, nblocks, T, dsa::kBlockTopk, blocks, dev->sm_count, stream)) != cudaSuccess)
    return cuda_fail(e, "block top-k launch");
  if ((e = dsa::launch_block_expand(blocks, n_vis, T, L.wa, idx_loc, idx_anc, idx_dyn, stream)) != cudaSuccess)
    return cuda_fail(e, "block index launch");
  const size_t tl = size_t(T) * DSA_HEADS;
  dsa::MlaLaunch pl{q,     kv,  cache_rows, kv_start,     idx_loc,       T,     dsa::kLocalWidth, scale,
                    o_loc, lse, part,       L.part_bytes, dev->sm_count, wait_limit_ns(), stream};
  if ((rc = run_sparse_mla(pl))) return rc;
  dsa::MlaLaunch pa{q,     kv,  cache_rows, kv_start, idx_anc, T, L.wa, scale, o_anc, lse ? lse + tl : nullptr, part,
                    L.part_bytes, dev->sm_count, wait_limit_ns(), stream};
  if ((rc = run_sparse_mla(pa))) return rc;
  dsa::MlaLaunch pd{q,     kv,  cache_rows, kv_start, idx_dyn, T, dsa::kDynWidth, scale, o_lat,
                    lse ? lse + 2 * tl : nullptr, part, L.part_bytes, dev->sm_count, wait_limit_ns(), stream};
  if ((rc = run_sparse_mla(pd))) return rc;
  if ((e = dsa::launch_fuse3(o_lat, o_loc, o_anc, gates, T, dev->sm_count, stream)) != cudaSuccess)
    return cuda_fail(e, "fusion launch");
  return DSA_OK;
}

int dsa_indexer_scores_noalloc(const dsa_bf16* q_I, const dsa_bf16* w, const dsa_bf16* k_I, int64_t cache_rows,
                               const int64_t* kv_start, const int32_t* n_vis, int T, float* scores, int64_t score_ld,
                               dsa_stream_t stream) {
  t_err.clear();
  int rc = check_common_rows(T, cache_rows, kv_start);
  if (rc) return rc;
  if (T > DSA_NOALLOC_MAX_ROWS)
    return fail(DSA_ERR_INVALID_ARG, "dsa_indexer_scores_noalloc handles at most %d query rows (got %d)",
                DSA_NOALLOC_MAX_ROWS, T);
  if (T == 0) return DSA_OK;
  if (!q_I || !w || !k_I || !n_vis || !scores) return fail(DSA_ERR_INVALID_ARG, "a required pointer is NULL");
  if (!aligned(q_I, 16) || !aligned(w, 16) || !aligned(k_I, 16) || !aligned(scores, 16) || !aligned(n_vis, 4))
    return fail(DSA_ERR_INVALID_ARG, "q_I, w, k_I, scores must be 16-byte aligned and n_vis 4-byte aligned");
  if (score_ld < 4 || score_ld % 4 != 0) return fail(DSA_ERR_INVALID_ARG, "score_ld must be a positive multiple of 4");
  DeviceState* dev = nullptr;
  if ((rc = current_device(&dev))) return rc;
  void* plan = nullptr;
  {
    // Once per device, with that device current: the host-side name of the array
    // is not a device address, so ask the runtime for this device's copy.  Under
    // the device lock, so two threads making their first call race on nothing.
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (!dev->noalloc_plan) {
      void* ptr = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_plan);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(plan scratch)");
      dev->noalloc_plan = ptr;
    }
    plan = dev->noalloc_plan;
  }
  // The plan kernel rewrites every header and tile entry it uses, so the array
  // needs no clearing between calls.
  return run_indexer(q_I, w, k_I, cache_rows, kv_start, n_vis, T, scores, score_ld, plan, stream, dev->sm_count);
}

void dsa_set_wait_limit_ns(unsigned long long ns) { g_wait_limit_override.store(ns, std::memory_order_relaxed); }

int dsa_check_wait_timeout(dsa_stream_t stream) {
  t_err.clear();
  DeviceState* dev = nullptr;
  int rc = current_device(&dev);
  if (rc) return rc;
  wait_probe_kernel<<<1, 32, 0, stream>>>(dsa::WaitLimit{wait_limit_ns()});
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "wait probe launch");
  return DSA_OK;
}

int dsa_sync_status(dsa_stream_t stream) {
  t_err.clear();
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int st = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&st, dsa::g_status, sizeof st);
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (st) {
    e = cudaMemcpyToSymbol(dsa::g_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  }
  if (st & dsa::kStatusTimeout) return fail(DSA_ERR_TIMEOUT, "a bounded device wait expired (status 0x%x)", st);
  if (st & (dsa::kStatusBadRow | dsa::kStatusOverflow))
    return fail(DSA_ERR_BAD_ROW, "a row was skipped: n_vis, kv_start or an index out of range (status 0x%x)", st);
  return DSA_OK;
}

}  // extern "C"
