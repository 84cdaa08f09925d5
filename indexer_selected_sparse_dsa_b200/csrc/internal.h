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
};
constexpr int kStreamCap = 8192;

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

// Shared-memory opt-in sizes, set once per device.
cudaError_t prepare_indexer();
cudaError_t prepare_sparse_mla();
cudaError_t prepare_topk();

}  // namespace dsa
