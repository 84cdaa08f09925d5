// Internal launch interface between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace dsa {

// ------------------------------------------------------------------ indexer plan
// A query tile is a run of <= qmax consecutive rows that read the same sequence
// (equal kv_start).  Its "units" are 128-key tiles of that sequence, enough to
// cover the largest n_vis in the tile.
struct PlanHeader {
  long long total_units;
  int n_tiles;
  int pad;
  long long pad2[2];
};
struct PlanTile {
  int q0;
  int nq;
  int units;
  int pad;
  long long kv_start;
  long long unit_begin;
};
static_assert(sizeof(PlanHeader) == 32, "plan header");
static_assert(sizeof(PlanTile) == 32, "plan tile");

inline size_t indexer_plan_bytes(int T) { return sizeof(PlanHeader) + sizeof(PlanTile) * size_t(T > 0 ? T : 1); }

enum SweepMode : int {
  kSweepSplit = 0,  // all units split evenly over the persistent CTAs
  kSweepWave = 1,   // CTA c takes whole query tiles c, c+G, ... (shared-key L2 reuse)
};

// Streaming selection (no score matrix): per query row a candidate buffer of
// `cap` (order key, position) pairs; the kept positions go to idx[T, topk].
struct StreamOut {
  uint32_t* cand_key;  // [T, cap]
  int32_t* cand_pos;   // [T, cap]
  int32_t* idx;        // [T, topk]
  int topk;
  int cap;
  // Threshold seeding: before its sweep, a long query tile scores sample_units
  // key units spread over its range and starts each query's filter at a
  // threshold that about (1 + 4 / sqrt(share)) x topk of its keys pass
  // (sample_mode 2: at the sample's maximum, which lets too few pass; a test
  // of the redo pass).  A query with fewer than topk passing keys at the end
  // is listed in redo[1 + i] (redo[0] counts them) and swept again unseeded.
  int* redo;           // [1 + T]
  int* cnt_out;        // [T]: candidates left in a query's buffer after its sweep (-1: none yet)
  int sample_units;
  int sample_mode;
};
constexpr int kStreamCap = 8192;
constexpr int kSampleUnits = 64;        // 8192 keys: fits the candidate buffer
constexpr int kSampleMinUnits = 1024;   // tiles of at least 128K keys are seeded

struct IndexerLaunch {
  const uint16_t* q_I;
  const uint16_t* w;
  const uint16_t* k_I;
  int64_t cache_rows;
  const int64_t* kv_start;
  const int32_t* n_vis;
  int T;
  float* scores;
  int64_t score_ld;
  void* plan;  // indexer_plan_bytes(T) bytes
  int qmax;    // 1, 4 or 8
  int sweep;   // SweepMode
  bool streaming;  // select into stream_out instead of writing scores (wave sweep, qmax 8)
  StreamOut stream_out;
  int grid;    // persistent CTAs
  unsigned long long wait_ns;
  cudaStream_t stream;
};
cudaError_t launch_indexer(const IndexerLaunch& p, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q);

// ------------------------------------------------------------------ top-k
// Rows longer than a few chunks are split over a cluster of up to 4 CTAs when
// there are fewer rows than SMs.
cudaError_t launch_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk,
                        int32_t* idx, int sm_count, cudaStream_t stream);

// ------------------------------------------------------------------ sparse MLA
struct MlaLaunch {
  const uint16_t* q;   // [T,64,576]: read through a tensor map (64-row boxes)
  const uint16_t* kv;  // [cache_rows,576]: gathered with 16-byte cp.async
  int64_t cache_rows;
  const int64_t* kv_start;
  const int32_t* idx;
  int T;
  int topk;
  float scale;
  float* o_lat;
  float* lse;
  float* part;        // split partials (may be null: one CTA per row)
  size_t part_bytes;
  int sm_count;
  unsigned long long wait_ns;
  cudaStream_t stream;
};
cudaError_t launch_sparse_mla(const MlaLaunch& p, const CUtensorMap& tmap_q);

// ------------------------------------------------------------------ dense + sparse branches
cudaError_t launch_window_idx(const int32_t* n_vis, int T, int window, int32_t* idx_w, cudaStream_t stream);
cudaError_t launch_fuse(float* o, const float* o_dense, const float* gate, int T, int sm_count, cudaStream_t stream);

// ------------------------------------------------------------------ block-level variant
constexpr int kBlockTokens = 128;                     // tokens per block
constexpr int kBlockTopk = 16;                        // dynamic branch: blocks per query
constexpr int kAnchorEvery = 16;                      // one anchor block in every 16
constexpr int kLocalWidth = 3 * kBlockTokens;         // local branch list: the query's block and its neighbours
constexpr int kDynWidth = kBlockTopk * kBlockTokens;  // dynamic branch list
cudaError_t launch_block_max(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int bld,
                             float* bscore, int32_t* nblocks, cudaStream_t stream);
cudaError_t launch_block_expand(const int32_t* blocks, const int32_t* n_vis, int T, int wa, int32_t* idx_loc,
                                int32_t* idx_anc, int32_t* idx_dyn, cudaStream_t stream);
cudaError_t launch_fuse3(float* o, const float* o_loc, const float* o_anc, const float* gates, int T, int sm_count,
                         cudaStream_t stream);

// ------------------------------------------------------------------ fused decode step
// The whole step of a batch of at most kDecodeMaxRows query rows in one
// cooperative launch (one CTA per SM): indexer, exact top-k, attention, merge.
constexpr int kDecodeMaxRows = 8;
constexpr int kDecodeTileRows = 4;      // query rows per indexer tile
constexpr int kDecodeMaxN = 32768;      // longest visible context (the row's scores sit in shared memory)
struct DecodeFusedLaunch {
  const uint16_t* w;
  const uint16_t* kv;
  const int64_t* kv_start;
  const int32_t* n_vis;
  int T;
  int topk;
  int64_t cache_rows;
  int64_t score_ld;
  float scale;
  float* scores;      // [T, score_ld]
  void* cand;         // [T, score_ld] pairs of (order key, position) that do not fit in shared memory
  uint32_t* sync;     // handoff counters, zeroed before each launch
  float* part;        // per attention tile: O (64 x 512), max, sum
  float* o_lat;
  float* lse;
  int32_t* idx;
  int sm_count;
  unsigned long long wait_ns;
  cudaStream_t stream;
};
cudaError_t launch_decode_fused(const DecodeFusedLaunch& p, const CUtensorMap& tmap_k, const CUtensorMap& tmap_qi,
                                const CUtensorMap& tmap_q);

// Shared-memory opt-in sizes, set once per device.
cudaError_t prepare_indexer();
cudaError_t prepare_sparse_mla();
cudaError_t prepare_topk();
cudaError_t prepare_decode_fused();
// Exact top-k of each query's candidate buffer (after the streamed sweep),
// written ascending and -1 padded; rows with cnt_out < 0 are left as they are.
cudaError_t launch_stream_select(const StreamOut& so, const int32_t* n_vis, int T, cudaStream_t stream);

}  // namespace dsa
