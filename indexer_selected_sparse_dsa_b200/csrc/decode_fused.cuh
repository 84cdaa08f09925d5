// The whole decode step of a small batch in one persistent launch.
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.2: a decode query is scored against its whole history by the
// lightning indexer but attends at most index_topk = 2048 positions.  With a
// few query rows the step moves only a few MB, so the separate kernels'
// launch, ramp and drain times, not bytes, set its length.)
//
// One cooperative launch of one CTA per SM (256 threads) runs four phases with
// grid-wide handoffs (release / acquire on a counter in the workspace, zeroed
// by a memset before the launch; every wait is bounded):
//  1. indexer: the batch's 128-key units split evenly over the CTAs.  TMA
//     brings each unit's keys (two-stage ring) and the query tile's q_I;
//     tcgen05 computes every head's dot product for up to 4 queries
//     (M = 128 keys, N = 32 x queries); the epilogue weights and sums the
//     heads per key and writes the scores to the workspace.
//  -- handoff --
//  2. selection, one CTA per query (CTAs that hold no attention tile): the
//     exact top-k of the query's scores, copied into shared memory.  The keys
//     of two ranks among 2048 strided scores give a window of order keys that
//     should hold the k-th score; one pass keeps the scores above the window
//     (a bitmap word per 32 positions, built from warp ballots), and bins and
//     lists those inside it; the bin of the k-th score is found by a scan and
//     its few entries ranked by (score, lower position first).  When the
//     window misses, an exact radix select over the whole row (per-warp
//     histograms of 11-bit key prefixes, then the remaining key bits, then
//     positions for ties) decides instead.  The bitmap's popcount scan
//     writes the kept positions in ascending order (the idx output).
//  -- handoff --
//  3. attention, one CTA per (query, 128-position tile of its kept list):
//     gather the tile's latent rows with 16-byte cp.async into the
//     128B-swizzled layout, S^T = K.Q^T on the tensor cores (q was prefetched
//     by TMA when the kernel started), the tile's softmax, O^T = V^T.P^T with
//     P (bf16) written over the rope chunk the score product no longer needs.
//     O is stored from the registers the TMEM loads fill: the output itself
//     for a one-tile query, else the tile's unnormalised O with its max and sum.
//  -- handoff (only when a query has several tiles) --
//  4. merge: one warp per (query, head, 128 latent dims) combines the tiles.
// The selection follows the top-k kernels' rule (scores ranked by value, ties
// to the lower position), taken on this kernel's own fp32 scores.
#pragma once
#include <cuda.h>

#include "block_scan.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFBinBits = 11;
constexpr int kFBins = 1 << kFBinBits;        // histogram bins
constexpr int kFBinShift = 32 - kFBinBits;    // bin = order key >> 21
constexpr int kFStages = 2;                   // key stages of the indexer ring
constexpr int kFKeyStage = 128 * 128 * 2;     // 32 KB: 128 keys x 128 dims
constexpr int kFQiBox = 32 * 64 * 2;          // 4 KB: one query's 32 heads, one 64-column half
constexpr int kFChunk = 128 * 128;            // 16 KB: 128 rows x 64 columns (bf16), 128B-swizzled
constexpr int kFQChunk = 64 * 128;            // 8 KB: 64 heads x 64 columns
constexpr int kFPartFloats = 64 * 512 + 2 * 64;  // one tile's O, max (log2 units), sum

// Shared memory, from the 1 KB-aligned base.
constexpr int kFQOff = 0;                        // attention q: 9 x 8 KB
constexpr int kFTileOff = 9 * kFQChunk;          // 73728: 144 KB shared by the phases
constexpr int kFTileBytes = 9 * kFChunk;
// phase 1 inside the tile region
constexpr int kFKeyOff = kFTileOff;                               // 2 x 32 KB key stages
constexpr int kFQiOff = kFKeyOff + kFStages * kFKeyStage;         // q_I tile: [half][4 queries] x 4 KB
static_assert(kFQiOff + 2 * kDecodeTileRows * kFQiBox <= kFTileOff + kFTileBytes, "phase-1 buffers");
// phase 2 (selection CTAs hold no attention tile: all of [0, kFMiscOff) is theirs):
// the row's scores, its bitmap, the tie list, the window list (or, on the slow
// path, one histogram per warp), the window histogram
constexpr int kFSelScoreOff = 0;                                  // kDecodeMaxN floats (128 KB)
constexpr int kFSelBitmapOff = kFSelScoreOff + kDecodeMaxN * 4;   // 131072
constexpr int kFSelTieOff = kFSelBitmapOff + kDecodeMaxN / 8;     // 135168
constexpr int kFSelTieCap = 256;
constexpr int kFSelWinOff = 147456;
constexpr int kFSelWinCap = 8192;                                 // (key, position) pairs (64 KB)
constexpr int kFSelWinPerWarp = kFSelWinCap / kFWarps;            // each warp's region of the window list
constexpr int kFSelWinHistOff = kFSelWinOff + kFSelWinCap * 8;    // 212992: 2048 bins
// everything else
constexpr int kFMiscOff = kFTileOff + kFTileBytes;  // 221184
static_assert(kFSelTieOff + kFSelTieCap * 8 <= kFSelWinOff, "selection buffers");
static_assert(kFSelWinHistOff + kFBins * 4 <= kFMiscOff, "selection buffers");
static_assert(kFWarps * kFBins * 4 <= kFSelWinCap * 8, "slow-path histograms");
constexpr int kFRedOff = kFMiscOff;                 // float red[4][64]
constexpr int kFMOff = kFRedOff + 1024;             // float m[64]  (log2 units)
constexpr int kFLOff = kFMOff + 256;                // float l[64]
constexpr int kFWOff = kFLOff + 256;                // float w[4][32]
constexpr int kFPosOff = kFWOff + 512;              // int pos[128]

struct FRow {
  long long ks;  // kv_start
  int n;         // n_vis (0: the row is skipped)
  int k;         // kept positions: min(topk, n)
  int tiles;     // attention tiles: ceil(k / 128)
  int att0;      // first attention unit of the row
};
struct FTile {
  long long ks;
  int q0, nq, units, unit_begin;
};
struct FPlan {
  FRow row[kDecodeMaxRows];
  FTile tile[kDecodeMaxRows];
  long long ks_in[kDecodeMaxRows];
  int n_in[kDecodeMaxRows];
  int n_tiles, total_units, att_units, multi;
};
constexpr int kFPlanOff = kFPosOff + 512;
constexpr int kFScanOff = (kFPlanOff + int(sizeof(FPlan)) + 15) & ~15;  // int scan[40]
constexpr int kFSelOff = kFScanOff + 160;                               // int sel[16]
constexpr int kFBarOff = (kFSelOff + 64 + 7) & ~7;
constexpr int kFNumBars = 17;
constexpr int kFSlotOff = kFBarOff + kFNumBars * 8;  // tmem slot, abort flag, phase-3 outcome
constexpr int kFSmemBytes = kFSlotOff + 16;
constexpr int kFSmemAlloc = kFSmemBytes + 1024;
constexpr uint32_t kFTmemCols = 512;
constexpr uint32_t kFSCol = 0;    // S^T: 64 columns (phase 3)
constexpr uint32_t kFOCol = 256;  // O^T: 4 x 64 columns (phase 3)

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add_u32(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// A CTA barrier reached with the warp converged first (role code leaves some lanes behind).
__device__ __forceinline__ void cta_sync() {
  __syncwarp();
  __syncthreads();
}

// hist[bin] += 1 for every lane with `active`, one shared atomic per distinct bin of
// the warp (scores cluster in a few bins; plain atomics would serialise on them).
__device__ __forceinline__ void warp_hist_add(uint32_t* hist, int bin, bool active) {
  const unsigned act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const unsigned peers = __match_any_sync(act, bin);
  if ((threadIdx.x & 31) == __ffs(int(peers)) - 1) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}

__device__ __forceinline__ uint32_t f_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Grid-wide handoff: each CTA adds one to *ctr with release semantics after its
// writes (the CTA barrier before it makes every thread's writes part of that
// release) and waits, with acquire loads, until all G have.  A CTA arrives even
// when it has aborted, so no other CTA waits for it; its own wait gives up
// after the limit (raising the timeout bit).
__device__ __forceinline__ bool grid_handoff(uint32_t* ctr, uint32_t G, WaitLimit lim, volatile int* abort_flag) {
  cta_sync();
  if (threadIdx.x == 0) {
    red_release_add_u32(ctr, 1u);
    if (ld_acquire_u32(ctr) < G) {
      const unsigned long long t0 = globaltimer();
      for (uint32_t it = 1;; ++it) {
        if (ld_acquire_u32(ctr) >= G) break;
        if ((it & 63u) == 0u && globaltimer() - t0 > lim.ns) {
          raise_status(kStatusTimeout);
          *abort_flag = 1;
          break;
        }
      }
    }
  }
  cta_sync();
  return *abort_flag == 0;
}

// One pass of a block-wide radix select over n items: counts digit(j) for the
// items with match(j) into hist[0, nbins) and finds the digit d, counted from the
// top, where the items above d number fewer than `need` and those at or above d
// at least `need`.  Returns d; *need becomes need minus the items above d and
// *eq the items on d.  nbins is a multiple of 256; all threads call it.
template <class Match, class Digit>
__device__ int block_select_pass(int n, int nbins, int* need, int* eq, uint32_t* hist, int* scan, int* res,
                                 Match match, Digit digit) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nbins; i += kFThreads) hist[i] = 0u;
  cta_sync();
  for (int j0 = 0; j0 < n; j0 += kFThreads) {  // whole warps per step: the adds are warp-aggregated
    const int j = j0 + tid;
    const bool act = j < n && match(j);
    warp_hist_add(hist, act ? digit(j) : 0, act);
  }
  cta_sync();
  const int per = nbins / kFThreads;
  int local = 0;
  for (int b = 0; b < per; ++b) local += int(hist[tid * per + b]);
  int total = 0;
  const int excl = block_exclusive_sum<int>(local, scan, &total);
  int above = total - excl - local;  // items in the bins of higher threads
  const int nd = *need;
  if (above < nd && above + local >= nd) {
    for (int b = per - 1; b >= 0; --b) {
      const int c = int(hist[tid * per + b]);
      if (above + c >= nd) {
        res[0] = tid * per + b;
        res[1] = nd - above;
        res[2] = c;
        break;
      }
      above += c;
    }
  }
  cta_sync();
  const int d = res[0];
  *need = res[1];
  *eq = res[2];
  cta_sync();
  return d;
}

struct FusedDecodeArgs {
  const uint16_t* w;       // [T,32]
  const uint16_t* kv;      // [cache_rows,576]
  const int64_t* kv_start;
  const int32_t* n_vis;
  int T;
  int topk;
  int64_t cache_rows;
  int64_t ld;              // score row stride (and candidate list capacity)
  float scale_log2;
  float* scores;           // [T, ld]
  uint2* cand;             // [T, ld]: candidates that do not fit in shared memory
  uint32_t* sync;          // handoff counters
  float* part;             // [att_units, kFPartFloats]
  float* o_lat;
  float* lse;
  int32_t* idx;            // [T, topk]
  WaitLimit lim;
};

__global__ void __launch_bounds__(kFThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_qi,
                        const __grid_constant__ CUtensorMap tmap_q, FusedDecodeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // 1 KB-aligned base by pointer arithmetic on the shared array (an integer round trip
  // would hide the shared address space and turn every access into a generic one)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float* red = reinterpret_cast<float*>(smem + kFRedOff);
  float* m_s = reinterpret_cast<float*>(smem + kFMOff);
  float* l_s = reinterpret_cast<float*>(smem + kFLOff);
  float* w_s = reinterpret_cast<float*>(smem + kFWOff);
  int* pos_s = reinterpret_cast<int*>(smem + kFPosOff);
  FPlan& plan = *reinterpret_cast<FPlan*>(smem + kFPlanOff);
  int* scan = reinterpret_cast<int*>(smem + kFScanOff);
  int* sel = reinterpret_cast<int*>(smem + kFSelOff);
  const uint32_t bar0 = sbase + kFBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };                 // 0, 1
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 + s); };          // 2, 3
  const uint32_t qi_full = bar0 + 8u * 4;
  const uint32_t qi_empty = bar0 + 8u * 5;
  auto afull_bar = [&](int b) { return bar0 + 8u * (6 + b); };          // 6, 7
  auto aempty_bar = [&](int b) { return bar0 + 8u * (8 + b); };         // 8, 9
  const uint32_t q_full = bar0 + 8u * 10;
  const uint32_t s_full = bar0 + 8u * 11;
  const uint32_t p_full = bar0 + 8u * 12;
  const uint32_t o_full = bar0 + 8u * 13;
  const uint32_t drain1 = bar0 + 8u * 14;
  const uint32_t drain3 = bar0 + 8u * 15;
  const uint32_t sel_bar = bar0 + 8u * 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kFSlotOff + 4);
  volatile int* att_ok = reinterpret_cast<volatile int*>(smem + kFSlotOff + 8);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = int(gridDim.x);
  const WaitLimit lim = a.lim;

  if (tid < a.T) {  // the rows' bounds, read in parallel
    plan.ks_in[tid] = a.kv_start[tid];
    plan.n_in[tid] = a.n_vis[tid];
  }
  if (tid == 64) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(qi_full, 1);
    mbar_init(qi_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(afull_bar(b), 1);
      mbar_init(aempty_bar(b), 4);  // one arrival per epilogue warp
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_full, 1);
    mbar_init(drain1, 1);
    mbar_init(drain3, 1);
    mbar_init(sel_bar, 1);
    *abort_flag = 0;
    *att_ok = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_qi);
    prefetch_tmap(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kFTmemCols);
    tmem_relinquish();
  }
  cta_sync();
  if (tid == 0) {
    // The plan, the same in every CTA: query tiles of up to 4 consecutive rows
    // reading the same sequence, their key units, and the attention units.
    int nt = 0, U = 0, A = 0, multi = 0;
    for (int r = 0; r < a.T; ++r) {
      FRow& R = plan.row[r];
      const long long ks = plan.ks_in[r];
      const int n = plan.n_in[r];
      const bool ok = n >= 1 && n <= a.ld && ks >= 0 && ks + n <= a.cache_rows;
      if (!ok && blockIdx.x == 0) raise_status(kStatusBadRow);
      R.ks = ok ? ks : 0;
      R.n = ok ? n : 0;
      R.k = ok ? min(a.topk, n) : 0;
      R.tiles = (R.k + 127) / 128;
      R.att0 = A;
      A += R.tiles;
      multi |= R.tiles > 1 ? 1 : 0;
      if (!ok) continue;
      const int units = (n + 127) / 128;
      FTile* last = nt > 0 ? &plan.tile[nt - 1] : nullptr;
      if (last && last->ks == ks && last->q0 + last->nq == r && last->nq < kDecodeTileRows) {
        ++last->nq;
        last->units = max(last->units, units);
      } else {
        FTile& t = plan.tile[nt++];
        t.ks = ks;
        t.q0 = r;
        t.nq = 1;
        t.units = units;
      }
    }
    for (int t = 0; t < nt; ++t) {
      plan.tile[t].unit_begin = U;
      U += plan.tile[t].units;
    }
    plan.n_tiles = nt;
    plan.total_units = U;
    plan.att_units = A;
    plan.multi = multi;
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // this CTA's key units [ub, ue), attention unit (row ra, tile ja), selection row rs
  const long long U = plan.total_units;
  const int ub = int(U * blockIdx.x / G), ue = int(U * (blockIdx.x + 1) / G);
  int ra = -1, ja = 0;
  if (int(blockIdx.x) < plan.att_units)
    for (int r = 0; r < a.T; ++r)
      if (int(blockIdx.x) >= plan.row[r].att0 && int(blockIdx.x) < plan.row[r].att0 + plan.row[r].tiles) {
        ra = r;
        ja = int(blockIdx.x) - plan.row[r].att0;
      }
  const int rs = G - 1 - int(blockIdx.x) < a.T ? G - 1 - int(blockIdx.x) : -1;
  auto tile_of = [&](int g, int t) {  // the tile holding unit g, searching from tile t
    while (g >= plan.tile[t].unit_begin + plan.tile[t].units) ++t;
    return t;
  };

  // ================================================================ phase 1: indexer
  if (warp == 0) {
    if (lane == 0) {
      int stage = 0, t = 0, prev = -1, issued[kFStages] = {0, 0}, qi_loads = 0;
      uint32_t ph = 0;
      bool q_issued = false;
      auto issue_q = [&]() {  // the attention phase's q, fetched during the indexer
        if (ra >= 0 && !q_issued) {
          mbar_arrive_expect_tx(q_full, 9 * kFQChunk);
          for (int c = 0; c < 9; ++c) tma_load_2d(sbase + kFQOff + c * kFQChunk, &tmap_q, q_full, 64 * c, ra * 64);
        }
        q_issued = true;
      };
      for (int g = ub; g < ue; ++g) {
        if (g == ub + kFStages) issue_q();  // behind the first key stages
        t = tile_of(g, t);
        const FTile& T0 = plan.tile[t];
        if (t != prev) {
          if (!mbar_wait(qi_empty, uint32_t(qi_loads & 1) ^ 1u, lim, abort_flag)) break;
          mbar_arrive_expect_tx(qi_full, uint32_t(T0.nq) * 2u * kFQiBox);
          for (int qi = 0; qi < T0.nq; ++qi) {
            const int y = (T0.q0 + qi) * 32;
            tma_load_2d(sbase + kFQiOff + qi * kFQiBox, &tmap_qi, qi_full, 0, y);
            tma_load_2d(sbase + kFQiOff + (kDecodeTileRows + qi) * kFQiBox, &tmap_qi, qi_full, 64, y);
          }
          ++qi_loads;
          prev = t;
        }
        if (!mbar_wait(empty_bar(stage), ph ^ 1u, lim, abort_flag)) break;
        mbar_arrive_expect_tx(full_bar(stage), kFKeyStage);
        const int y = int(T0.ks + (long long)(g - T0.unit_begin) * 128);
        const uint32_t kdst = sbase + kFKeyOff + stage * kFKeyStage;
        tma_load_2d(kdst, &tmap_k, full_bar(stage), 0, y);
        tma_load_2d(kdst + kFKeyStage / 2, &tmap_k, full_bar(stage), 64, y);
        ++issued[stage];
        if (++stage == kFStages) {
          stage = 0;
          ph ^= 1u;
        }
      }
      issue_q();
      // every copy issued above lands before its buffer is reused or the CTA exits
      for (int s = 0; s < kFStages; ++s)
        if (issued[s] > 0) mbar_drain(full_bar(s), uint32_t((issued[s] - 1) & 1));
      if (qi_loads > 0) mbar_drain(qi_full, uint32_t((qi_loads - 1) & 1));
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0, t = 0, prev = -1, ab = 0, qi_loads = 0;
      uint32_t ph = 0, aph = 0;
      for (int g = ub; g < ue; ++g) {
        t = tile_of(g, t);
        const int nq = plan.tile[t].nq;
        if (t != prev) {
          if (prev >= 0) mma_commit(qi_empty);  // the previous tile's q_I is free once its MMAs finish
          if (!mbar_wait(qi_full, uint32_t(qi_loads & 1), lim, abort_flag)) break;
          ++qi_loads;
          prev = t;
        }
        if (!mbar_wait(aempty_bar(ab), aph ^ 1u, lim, abort_flag)) break;
        if (!mbar_wait(full_bar(stage), ph, lim, abort_flag)) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 32 * nq, 0, 0);
        const uint32_t kaddr = sbase + kFKeyOff + stage * kFKeyStage;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t koff = uint32_t((k >> 2) * (kFKeyStage / 2) + (k & 3) * 32);
          const uint32_t qoff = uint32_t((k >> 2) * kDecodeTileRows * kFQiBox + (k & 3) * 32);
          const uint64_t ad = smem_desc(kaddr + koff, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(sbase + kFQiOff + qoff, 16, 1024, kSwizzle128B);
          mma_bf16_ss(tmem + uint32_t(ab * 128), ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(empty_bar(stage));
        mma_commit(afull_bar(ab));
        if (++stage == kFStages) {
          stage = 0;
          ph ^= 1u;
        }
        if (++ab == 2) {
          ab = 0;
          aph ^= 1u;
        }
      }
      mma_commit(drain1);  // every MMA above has completed before TMEM is reused
      mbar_drain(drain1, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // epilogue: thread = key row (TMEM lane) of the unit
    const int et = tid - 128, qw = warp & 3, kr = qw * 32 + lane;
    const uint32_t lane_addr = tmem + (uint32_t(qw * 32) << 16);
    int t = 0, prev = -1, ab = 0;
    uint32_t aph = 0;
    bool alive = true;
    for (int g = ub; g < ue; ++g) {
      t = tile_of(g, t);
      const FTile& T0 = plan.tile[t];
      if (t != prev) {
        named_bar_sync(1, 128);
        for (int e = et; e < T0.nq * 32; e += 128) w_s[e] = bf16_bits_to_float(a.w[(long long)T0.q0 * 32 + e]);
        named_bar_sync(1, 128);
        prev = t;
      }
      if (alive) alive = __all_sync(0xffffffffu, mbar_wait(afull_bar(ab), aph, lim, abort_flag));
      if (alive) {
        tc_fence_after();
        const int pos = (g - T0.unit_begin) * 128 + kr;
        for (int j = 0; j < T0.nq; ++j) {
          float v[32];
          tmem_ld32_sync(lane_addr + uint32_t(ab * 128 + 32 * j), v);
          float s = 0.f;
#pragma unroll
          for (int h = 0; h < 32; ++h) s = fmaf(w_s[32 * j + h], v[h], s);
          if (pos < plan.row[T0.q0 + j].n) a.scores[(long long)(T0.q0 + j) * a.ld + pos] = s;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(aempty_bar(ab));
      }
      if (++ab == 2) {
        ab = 0;
        aph ^= 1u;
      }
    }
  }
  grid_handoff(a.sync + 0, uint32_t(G), lim, abort_flag);

  // ================================================================ phase 2: exact top-k of one query
  if (rs >= 0 && plan.row[rs].n > 0 && *abort_flag == 0) {
    const FRow& R = plan.row[rs];
    const int n = R.n, k = R.k;
    int32_t* irow = a.idx + (long long)rs * a.topk;
    if (n <= a.topk) {
      for (int e = tid; e < a.topk; e += kFThreads) irow[e] = e < n ? e : -1;
    } else {
      const float* srow = a.scores + (long long)rs * a.ld;
      const int n4 = (n + 3) & ~3;  // whole float4s (the row stride is a multiple of 4)
      const int W = (n + 31) >> 5;
      float* sc = reinterpret_cast<float*>(smem + kFSelScoreOff);
      uint32_t* bm = reinterpret_cast<uint32_t*>(smem + kFSelBitmapOff);
      uint2* wl = reinterpret_cast<uint2*>(smem + kFSelWinOff);
      uint32_t* wh = reinterpret_cast<uint32_t*>(smem + kFSelWinHistOff);
      uint2* tl = reinterpret_cast<uint2*>(smem + kFSelTieOff);
      // (a) the row into shared memory by bulk copy; the bitmap and window histogram cleared
      if (tid == 0) {
        mbar_arrive_expect_tx(sel_bar, uint32_t(n4) * 4u);
        for (int off = 0; off < n4; off += 4096)
          bulk_load_g2s(sbase + kFSelScoreOff + 4u * uint32_t(off), srow + off, 4u * uint32_t(min(4096, n4 - off)),
                        sel_bar);
      }
      for (int w = tid; w < W; w += kFThreads) bm[w] = 0u;
      for (int b = tid; b < kFBins; b += kFThreads) wh[b] = 0u;
      if (tid < 8) sel[tid] = 0;
      if (tid == 0 && !mbar_wait(sel_bar, 0, lim, abort_flag)) mbar_drain(sel_bar, 0);
      cta_sync();
      // (b) a window [t_lo, t_hi] of order keys holding the k-th: the keys of ranks
      //     r_lo and r_hi among 2048 strided scores (exact: a bitwise radix over the
      //     CTA, each warp counting its 256 samples, one warp reduction and one CTA
      //     barrier per bit)
      uint32_t kv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int si = warp * 256 + lane + 32 * j;
        kv[j] = f_order_key(sc[(int)((long long)si * n / (kFWarps * 256))]);
      }
      const float sh = float(k) * float(kFWarps * 256) / float(n);  // the sample's expected share of the top k
      int r_lo = min(kFWarps * 256, int(ceilf(sh + 4.f * sqrtf(sh))) + 8);
      int r_hi = max(1, int(floorf(sh - 4.f * sqrtf(sh))) - 8);
      uint32_t t_lo = 0u, t_hi = 0u, mask = 0u;
      int* bits_s = reinterpret_cast<int*>(red);  // [2 parities][8 warps][2 ranks]
#pragma unroll 1
      for (int b = 31; b >= 0; --b) {
        const uint32_t bit = 1u << b, m2 = mask | bit, wa = t_lo | bit, wb = t_hi | bit;
        int ca = 0, cb = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          ca += (kv[j] & m2) == wa ? 1 : 0;
          cb += (kv[j] & m2) == wb ? 1 : 0;
        }
        ca = int(__reduce_add_sync(0xffffffffu, unsigned(ca)));
        cb = int(__reduce_add_sync(0xffffffffu, unsigned(cb)));
        int* slot = bits_s + (b & 1) * 2 * kFWarps;
        if (lane == 0) {
          slot[2 * warp] = ca;
          slot[2 * warp + 1] = cb;
        }
        __syncthreads();  // warps are converged here (every lane ran the reductions)
        int ta = 0, tb = 0;
#pragma unroll
        for (int w = 0; w < kFWarps; ++w) {
          ta += slot[2 * w];
          tb += slot[2 * w + 1];
        }
        if (ta >= r_lo) t_lo = wa;
        else r_lo -= ta;
        if (tb >= r_hi) t_hi = wb;
        else r_hi -= tb;
        mask = m2;
      }
      const uint32_t span = t_hi - t_lo;
      const int shift = 32 - __clz(int(span >> 11));  // the smallest shift with (span >> shift) < 2048
      // (c) one pass, 4 consecutive positions per thread: keys above t_hi are kept
      //     (bitmap words assembled from warp ballots, stored whole), keys in the
      //     window are counted in its histogram and appended to the warp's region
      //     of the window list (offsets from the ballots: no atomics, no scans)
      int gt = 0, woff = 0;
      const int wbase = warp * kFSelWinPerWarp;
      auto spread4 = [](uint32_t m) {  // bit l of an 8-bit mask to bit 4 l
        m = (m | (m << 12)) & 0x000F000Fu;
        m = (m | (m << 6)) & 0x03030303u;
        return (m | (m << 3)) & 0x11111111u;
      };
      for (int base = 0; base < n4; base += 4 * kFThreads) {
        const int p0 = base + 4 * tid;
        uint32_t kk[4] = {0u, 0u, 0u, 0u};
        if (p0 < n4) {
          const float4 v = *reinterpret_cast<const float4*>(sc + p0);
          kk[0] = f_order_key(v.x);
          kk[1] = f_order_key(v.y);
          kk[2] = f_order_key(v.z);
          kk[3] = f_order_key(v.w);
        }
        unsigned kb[4], wbl[4];
        int wrun = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const bool valid = p0 + q < n;
          const bool kept = valid && kk[q] > t_hi;
          const bool inw = valid && !kept && kk[q] >= t_lo;
          kb[q] = __ballot_sync(0xffffffffu, kept);
          wbl[q] = __ballot_sync(0xffffffffu, inw);
          gt += kept ? 1 : 0;
          if (inw) {
            const int slot = woff + wrun + __popc(wbl[q] & ((1u << lane) - 1u));
            if (slot < kFSelWinPerWarp) wl[wbase + slot] = make_uint2(kk[q], uint32_t(p0 + q));
            atomicAdd(&wh[(kk[q] - t_lo) >> shift], 1u);
          }
          wrun += __popc(wbl[q]);
        }
        woff += wrun;
        if (lane < 4) {  // word `lane` of the warp's 128 positions: lanes 8 lane .. 8 lane + 7
          uint32_t word = 0u;
#pragma unroll
          for (int q = 0; q < 4; ++q) word |= spread4((kb[q] >> (8 * lane)) & 0xFFu) << q;
          const int wi = (base >> 5) + 4 * warp + lane;
          if (wi < W) bm[wi] = word;
        }
      }
      if (lane == 0) sel[8 + warp] = woff;
      int gt_total = 0;
      (void)block_exclusive_sum<int>(gt, scan, &gt_total);
      int nw = 0;
      bool fits = true;
#pragma unroll
      for (int w = 0; w < kFWarps; ++w) {
        nw += sel[8 + w];
        fits = fits && sel[8 + w] <= kFSelWinPerWarp;
      }
      // (d) the window bin of the k-th key, counted from the top
      bool ok = fits && gt_total < k && gt_total + nw >= k;
      int bstar = 0, need = 0, eq = 0;
      {
        uint32_t cb[8];
        int local = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          cb[b] = wh[8 * tid + b];
          local += int(cb[b]);
        }
        int total = 0;
        const int excl = block_exclusive_sum<int>(local, scan, &total);
        int above = gt_total + (total - excl - local);
        if (ok && above < k && above + local >= k)
          for (int b = 7; b >= 0; --b) {
            if (above + int(cb[b]) >= k) {
              sel[1] = 8 * tid + b;
              sel[2] = k - above;
              sel[3] = int(cb[b]);
              break;
            }
            above += int(cb[b]);
          }
        cta_sync();
        bstar = sel[1];
        need = sel[2];
        eq = sel[3];
      }
      ok = ok && eq <= kFSelTieCap;
      if (ok) {
        // (e) window keys above the bin are kept; the bin's keys go to the tie list
        for (int j = tid; j < kFWarps * kFSelWinPerWarp; j += kFThreads) {
          if ((j % kFSelWinPerWarp) >= sel[8 + j / kFSelWinPerWarp]) continue;
          const uint2 e = wl[j];
          const int b = int((e.x - t_lo) >> shift);
          if (b > bstar) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
          else if (b == bstar) tl[atomicAdd(&sel[4], 1)] = e;
        }
        cta_sync();
        // (f) the bin's `need` best by (key descending, position ascending): each of its
        //     entries is kept when fewer than `need` entries beat it
        for (int j = tid; j < eq; j += kFThreads) {
          const uint2 e = tl[j];
          int beaten = 0;
          for (int i = 0; i < eq; ++i) {
            const uint2 f = tl[i];
            beaten += (f.x > e.x || (f.x == e.x && f.y < e.y)) ? 1 : 0;
          }
          if (beaten < need) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
        }
      } else {
        // The sample's window missed the k-th key or held too many keys: one
        // histogram per warp of the 11-bit key prefixes, then the bin's keys settled
        // by radix passes (exact; the slow path).
        uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kFSelWinOff);  // 8 x 2048, over the window list
        for (int w = tid; w < W; w += kFThreads) bm[w] = 0u;
        for (int e = tid; e < kFWarps * kFBins; e += kFThreads) hist[e] = 0u;
        if (tid == 0) sel[4] = 0;
        cta_sync();
        uint32_t* hw = hist + warp * kFBins;
        for (int base = 0; base < n; base += kFThreads) {
          const int p = base + tid;
          warp_hist_add(hw, p < n ? int(f_order_key(sc[p]) >> kFBinShift) : 0, p < n);
        }
        cta_sync();
        {
          uint32_t cb[8];
          int local = 0;
#pragma unroll
          for (int b = 0; b < 8; ++b) {
            uint32_t c = 0;
#pragma unroll
            for (int w = 0; w < kFWarps; ++w) c += hist[w * kFBins + 8 * tid + b];
            cb[b] = c;
            local += int(c);
          }
          int total = 0;
          const int excl = block_exclusive_sum<int>(local, scan, &total);
          int above = total - excl - local;
          if (above < k && above + local >= k) {
            for (int b = 7; b >= 0; --b) {
              if (above + int(cb[b]) >= k) {
                sel[0] = 8 * tid + b;
                sel[1] = k - above;
                sel[2] = int(cb[b]);
                break;
              }
              above += int(cb[b]);
            }
          }
          cta_sync();
        }
        const int bs = sel[0], need0 = sel[1], mb = sel[2];
        const bool cand_smem = mb <= kFSelWinCap;
        uint2* cf = cand_smem ? reinterpret_cast<uint2*>(hist) : a.cand + (long long)rs * a.ld;
        cta_sync();  // the histograms are read: their space takes the candidates
        for (int base = 0; base < n; base += kFThreads) {
          const int p = base + tid;
          const uint32_t key = p < n ? f_order_key(sc[p]) : 0u;
          const int bin = int(key >> kFBinShift);
          const bool kept = p < n && bin > bs;
          const bool cnd = p < n && bin == bs;
          const unsigned km = __ballot_sync(0xffffffffu, kept);
          if (lane == 0 && p < n) bm[p >> 5] = km;
          const unsigned cm = __ballot_sync(0xffffffffu, cnd);
          if (cm) {
            int basec = 0;
            if (lane == 0) basec = atomicAdd(&sel[4], __popc(cm));
            basec = __shfl_sync(0xffffffffu, basec, 0);
            if (cnd) {
              const int slot = basec + __popc(cm & ((1u << lane) - 1u));
              if (slot < mb) cf[slot] = make_uint2(key, uint32_t(p));
            }
          }
        }
        cta_sync();
        uint32_t kth = 0u;
        int pmax = 0x7fffffff;
        const bool all_cand = need0 >= mb;
        if (!all_cand) {
          int nd = need0, q = 0;
          const int d1 = block_select_pass(mb, 2048, &nd, &q, wh, scan, sel, [&](int) { return true; },
                                           [&](int j) { return int((cf[j].x >> 10) & 0x7ffu); });
          const int d2 = block_select_pass(mb, 1024, &nd, &q, wh, scan, sel,
                                           [&](int j) { return int((cf[j].x >> 10) & 0x7ffu) == d1; },
                                           [&](int j) { return int(cf[j].x & 0x3ffu); });
          kth = (uint32_t(bs) << kFBinShift) | (uint32_t(d1) << 10) | uint32_t(d2);
          if (nd < q) {  // only some tied keys fit: the lowest positions (21 bits) win
            const int p1 = block_select_pass(mb, 2048, &nd, &q, wh, scan, sel,
                                             [&](int j) { return cf[j].x == kth; },
                                             [&](int j) { return 0x7ff - int((cf[j].y >> 10) & 0x7ffu); });
            const int p2 = block_select_pass(
                mb, 1024, &nd, &q, wh, scan, sel,
                [&](int j) { return cf[j].x == kth && 0x7ff - int((cf[j].y >> 10) & 0x7ffu) == p1; },
                [&](int j) { return 0x3ff - int(cf[j].y & 0x3ffu); });
            pmax = ((0x7ff - p1) << 10) | (0x3ff - p2);
          }
        }
        for (int j = tid; j < mb; j += kFThreads) {
          const uint2 e = cf[j];
          const bool keep = all_cand || e.x > kth || (e.x == kth && int(e.y) <= pmax);
          if (keep && e.y < uint32_t(n)) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
        }
      }
      cta_sync();
      // (g) the kept positions in ascending order
      const int per = (W + kFThreads - 1) / kFThreads;
      const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
      int cnt = 0;
      for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
      int total = 0;
      int rank = block_exclusive_sum<int>(cnt, scan, &total);
      for (int w = w0; w < w1; ++w) {
        uint32_t bits = bm[w];
        while (bits) {
          const int b = __ffs(int(bits)) - 1;
          if (rank < a.topk) irow[rank] = 32 * w + b;
          ++rank;
          bits &= bits - 1u;
        }
      }
      for (int e = k + tid; e < a.topk; e += kFThreads) irow[e] = -1;
    }
  }
  grid_handoff(a.sync + 1, uint32_t(G), lim, abort_flag);

  // ================================================================ phase 3: attention of one tile
  if (ra >= 0) {
    const FRow& R = plan.row[ra];
    const bool live = *abort_flag == 0;
    if (tid < 128) pos_s[tid] = (live && 128 * ja + tid < R.k) ? a.idx[(long long)ra * a.topk + 128 * ja + tid] : -1;
    cta_sync();
    // gather the 128 latent rows: chunk c holds columns 64 c .. 64 c + 63, 128B-swizzled
    if (live) {
      const char* kvb = reinterpret_cast<const char*>(a.kv);
      for (int e = tid; e < 128 * 72; e += kFThreads) {
        const int rr = e / 72, gi = e - rr * 72, c = gi >> 3, g = gi & 7;
        int p = pos_s[rr];
        if (p >= R.n) p = -1;
        const uint32_t dst = sbase + kFTileOff + c * kFChunk + rr * 128 + ((g ^ (rr & 7)) << 4);
        const char* src = kvb + (R.ks + (p >= 0 ? p : 0)) * (576 * 2) + gi * 16;
        cp_async_16_or_zero(dst, src, p < 0);
      }
    }
    cp_async_wait_all();
    fence_proxy_async_smem();
    cta_sync();
    if (warp == 1) {
      // S^T = K.Q^T, then O^T = V^T.P^T
      if (lane == 0) {
        bool ok = *abort_flag == 0 && mbar_wait(q_full, 0, lim, abort_flag);
        if (ok) {
          tc_fence_after();
          const uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
          for (int c = 0; c < 9; ++c)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = smem_desc(sbase + kFTileOff + c * kFChunk + 32 * k, 16, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sbase + kFQOff + c * kFQChunk + 32 * k, 16, 1024, kSwizzle128B);
              mma_bf16_ss(tmem + kFSCol, ad, bd, idesc_s, (c | k) ? 1u : 0u);
            }
          mma_commit(s_full);
          ok = mbar_wait(p_full, 0, lim, abort_flag);
        }
        if (ok) {
          tc_fence_after();
          const uint32_t idesc_o = idesc_bf16(128, 64, 1, 1);
          for (int mm = 0; mm < 4; ++mm)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              // V^T: latent dims 128 mm .. 128 mm + 127 = chunks 2 mm, 2 mm + 1; keys 16 k .. 16 k + 15
              const uint64_t ad = smem_desc(sbase + kFTileOff + 2 * mm * kFChunk + k * 2048, kFChunk, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sbase + kFTileOff + 8 * kFChunk + k * 2048, kFChunk, 1024, kSwizzle128B);
              mma_bf16_ss(tmem + kFOCol + 64 * mm, ad, bd, idesc_o, k > 0 ? 1u : 0u);
            }
          mma_commit(o_full);
        }
        mma_commit(drain3);
        mbar_drain(drain3, 0);
      }
      __syncwarp();
    } else if (warp >= 4) {
      // softmax over the tile: thread = key row
      const int et = tid - 128, qw = warp & 3, kr = qw * 32 + lane;
      const uint32_t lane_addr = tmem + (uint32_t(qw * 32) << 16);
      auto wait_all = [&](uint32_t bar) {
        const bool mine = et == 0 ? mbar_wait(bar, 0, lim, abort_flag) : true;
        return bar_red_or_128(mine ? 0 : 1) == 0;
      };
      const bool valid = pos_s[kr] >= 0;
      bool ok = wait_all(s_full);
      if (ok) {
        tc_fence_after();
        float x[64];
        tmem_ld32_sync(lane_addr + kFSCol, x);
        tmem_ld32_sync(lane_addr + kFSCol + 32, x + 32);
#pragma unroll
        for (int h = 0; h < 64; ++h) x[h] = valid ? x[h] * a.scale_log2 : -INFINITY;
        float r0, r1;
        reduce_scatter64<true>(x, r0, r1);
        red[qw * 64 + 2 * lane] = r0;
        red[qw * 64 + 2 * lane + 1] = r1;
        named_bar_sync(1, 128);
        if (et < 64) m_s[et] = fmax_(fmax_(red[et], red[64 + et]), fmax_(red[128 + et], red[192 + et]));
        named_bar_sync(1, 128);
        uint8_t* prow = smem + kFTileOff + 8 * kFChunk + kr * 128;
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) {
          uint32_t w4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int h = gg * 8 + 2 * u;
            const float e0 = valid ? fast_exp2(x[h] - m_s[h]) : 0.f;
            const float e1 = valid ? fast_exp2(x[h + 1] - m_s[h + 1]) : 0.f;
            float q0, q1;
            w4[u] = pack_bf16x2(e0, e1, q0, q1);
            x[h] = q0;  // the sums take the rounded values the product uses
            x[h + 1] = q1;
          }
          *reinterpret_cast<uint4*>(prow + ((gg ^ (kr & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        reduce_scatter64<false>(x, r0, r1);
        red[qw * 64 + 2 * lane] = r0;
        red[qw * 64 + 2 * lane + 1] = r1;
        named_bar_sync(1, 128);
        if (et < 64) l_s[et] = red[et] + red[64 + et] + red[128 + et] + red[192 + et];
        ok = wait_all(o_full);
      }
      if (et == 0) *att_ok = ok ? 1 : 0;
      tc_fence_before();
    }
    cta_sync();
    // O^T out of TMEM (warps 0-3: latent dims 0-255, warps 4-7: 256-511), stored as
    // [head][512] floats (for a split row then its max and sum): a warp's store is
    // 32 consecutive latent dims of one head
    if (*att_ok) {
      tc_fence_after();
      const bool single = R.tiles == 1;
      float* dst = single ? a.o_lat + (long long)ra * 64 * 512 : a.part + (long long)blockIdx.x * kFPartFloats;
      const int qw = warp & 3;
      const uint32_t lane_addr = tmem + (uint32_t(qw * 32) << 16);
#pragma unroll 1
      for (int mi = 0; mi < 2; ++mi) {
        const int mm = 2 * (warp >> 2) + mi;
        const int d = 128 * mm + qw * 32 + lane;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float o[32];
          tmem_ld32_sync(lane_addr + kFOCol + 64 * mm + 32 * half, o);
#pragma unroll
          for (int hh = 0; hh < 32; ++hh) {
            const int h = 32 * half + hh;
            dst[h * 512 + d] = single ? o[hh] / l_s[h] : o[hh];
          }
        }
      }
      if (tid < 64) {
        if (single) {
          if (a.lse) a.lse[ra * 64 + tid] = (m_s[tid] + log2f(l_s[tid])) * 0.69314718055994531f;
        } else {
          dst[64 * 512 + tid] = m_s[tid];
          dst[64 * 512 + 64 + tid] = l_s[tid];
        }
      }
    }
  }

  // ================================================================ phase 4: merge the tiles
  if (plan.multi) {
    grid_handoff(a.sync + 2, uint32_t(G), lim, abort_flag);
    if (*abort_flag == 0)
      for (int p = int(blockIdx.x) * kFWarps + warp; p < a.T * 256; p += G * kFWarps) {
        const int r = p >> 8, h = (p >> 2) & 63, qd = p & 3;
        const FRow& R = plan.row[r];
        const int nt = R.tiles;
        if (nt <= 1) continue;
        const float* pb = a.part + (long long)R.att0 * kFPartFloats;
        const int d = 128 * qd + 4 * lane;
        float4 x[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (j < nt) x[j] = *reinterpret_cast<const float4*>(pb + (long long)j * kFPartFloats + h * 512 + d);
        const float mj = lane < nt ? pb[(long long)lane * kFPartFloats + 64 * 512 + h] : -INFINITY;
        const float lj = lane < nt ? pb[(long long)lane * kFPartFloats + 64 * 512 + 64 + h] : 0.f;
        float M = mj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmax_(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float wj = lane < nt ? fast_exp2(mj - M) : 0.f;
        float den = wj * lj;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
        const float inv = den > 0.f ? 1.f / den : 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float wt = __shfl_sync(0xffffffffu, wj, j);
          if (j < nt) {
            acc.x = fmaf(wt, x[j].x, acc.x);
            acc.y = fmaf(wt, x[j].y, acc.y);
            acc.z = fmaf(wt, x[j].z, acc.z);
            acc.w = fmaf(wt, x[j].w, acc.w);
          }
        }
        *reinterpret_cast<float4*>(a.o_lat + ((long long)r * 64 + h) * 512 + d) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (qd == 0 && lane == 0 && a.lse)
          a.lse[r * 64 + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
      }
  }

  // Skipped rows: zero output, lse -inf, no positions.
  if (blockIdx.x == gridDim.x - 1)
    for (int r = 0; r < a.T; ++r)
      if (plan.row[r].n == 0) {
        for (int e = tid; e < 64 * 512; e += kFThreads) a.o_lat[(long long)r * 64 * 512 + e] = 0.f;
        for (int e = tid; e < a.topk; e += kFThreads) a.idx[(long long)r * a.topk + e] = -1;
        if (a.lse && tid < 64) a.lse[r * 64 + tid] = -INFINITY;
      }

  // the attention's q copy lands before the CTA exits, even when nothing waited for it
  if (tid == 0 && ra >= 0) mbar_drain(q_full, 0);
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, kFTmemCols);
  }
}

}  // namespace

inline size_t decode_fused_sync_bytes() { return 64; }

cudaError_t prepare_decode_fused() {
  static_assert(kFSmemAlloc <= 232448, "fused decode shared memory exceeds the per-CTA limit");
  return cudaFuncSetAttribute(decode_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFSmemAlloc);
}

cudaError_t launch_decode_fused(const DecodeFusedLaunch& p, const CUtensorMap& tmap_k, const CUtensorMap& tmap_qi,
                                const CUtensorMap& tmap_q) {
  if (p.T <= 0) return cudaSuccess;
  if (p.T > kDecodeMaxRows) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(p.sync, 0, decode_fused_sync_bytes(), p.stream);
  if (e != cudaSuccess) return e;
  FusedDecodeArgs a{};
  a.w = p.w;
  a.kv = p.kv;
  a.kv_start = p.kv_start;
  a.n_vis = p.n_vis;
  a.T = p.T;
  a.topk = p.topk;
  a.cache_rows = p.cache_rows;
  a.ld = p.score_ld;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.scores = p.scores;
  a.cand = reinterpret_cast<uint2*>(p.cand);
  a.sync = p.sync;
  a.part = p.part;
  a.o_lat = p.o_lat;
  a.lse = p.lse;
  a.idx = p.idx;
  a.lim = WaitLimit{p.wait_ns};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(p.sm_count));
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = kFSmemAlloc;
  cfg.stream = p.stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: the handoffs wait on all of them
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_fused_kernel, tmap_k, tmap_qi, tmap_q, a);
}

}  // namespace dsa
