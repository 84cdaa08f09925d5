// Exact per-row top-k over materialised fp32 indexer scores.
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.2: keep the index_topk highest-scoring positions.  Ties go to the
// lower position; the kept positions are written in ascending order and padded
// with -1.)
//
// Scores map to 32-bit keys whose unsigned order is the float order (-0 is
// folded onto +0), so "k-th largest" is a radix select on keys.  One CTA of
// 1024 threads per row:
//   1. the first chunks of the row start streaming (16-byte cp.async into a
//      3-deep ring in shared memory; each thread reads back only its own
//      slots, so the ring needs no barrier) while a row longer than the
//      candidate buffer takes a strided sample of kSamples keys; two histogram
//      passes over the sample give a threshold tau_lo near its r-th largest
//      key, r a few standard deviations above the sample's expected share of k;
//   2. each thread tests its keys of a chunk against the current rule with
//      one float compare each; a warp scan places the passing keys, with their
//      positions, in the warp's own region of the shared candidate buffer (no
//      atomics, no order);
//   3. if a warp's region is full, the regions are gathered into one run and,
//      with more than k entries, cut to their exact top-k (ties to lower
//      positions); the rule tightens to "beats the worst kept entry", fresh
//      regions of >= one chunk's worth follow the kept run and the warps that
//      did not fit retry.  Every dropped entry has k better ones, so the
//      result stays exact;
//   4. an exact radix select over the candidates (12 + 10 + 10 bit
//      histograms; a second select over positions when the k-th key is tied)
//      fixes the kept set, which is written in ascending order through a
//      position bitmap in shared memory, one 131072-position window at a time.
// If fewer than k keys pass tau_lo (a sample far off its expectation) the row
// is redone by the full multi-pass radix select over global memory.
#pragma once
#include <climits>
#include <cstdlib>

#include "block_scan.cuh"
#include "dsa.h"
#include "internal.h"
#include "ptx.cuh"
#include "topk_short.cuh"

namespace dsa {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kSamplesPerThread = 4;
constexpr int kSamples = kTopkThreads * kSamplesPerThread;  // 4096
constexpr int kCandCap = 10240;                     // 320 per warp before any cut
constexpr int kHistBins = 4096;
constexpr int kChunkVec = 2;                        // float4 per thread per chunk
constexpr int kChunkF4 = kTopkThreads * kChunkVec;  // 2048 float4 = 8192 scores
constexpr int kKeysPerThread = kChunkVec * 4;
constexpr int kRing = 3;                            // chunks in flight
constexpr int kBitmapWords = 4096;                  // output window: 131072 positions
constexpr int kWordsPerThread = kBitmapWords / kTopkThreads;
static_assert(kWordsPerThread == 4, "bitmap words are read as one uint4 per thread");
static_assert((kCandCap - DSA_MAX_TOPK) / kTopkWarps >= 32 * kKeysPerThread, "after a cut every warp region takes a whole chunk");
static_assert(kBitmapWords * 4 <= kRing * kChunkF4 * 16, "the bitmap lives in the idle ring");

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose key is k, for comparing raw scores against a key threshold
// (x >= key_float(k) <=> order_key(x) >= k for every non-NaN x).  Keys below
// that of -inf belong to NaN bit patterns; -inf stands in for them.
__device__ __forceinline__ float key_float(uint32_t k) {
  if (k & 0x80000000u) return __uint_as_float(k & 0x7fffffffu);
  if (k <= 0x007fffffu) return __uint_as_float(0xff800000u);
  return __uint_as_float(~k);
}

struct TopkShared {
  float4 ring[kRing][kChunkF4];  // stream ring; the output bitmap once the stream is done
  uint32_t cand_key[kCandCap];
  int32_t cand_pos[kCandCap];
  uint32_t hist[kHistBins];
  int scan_i[33];
  int wsum[kTopkWarps];
  int sel_bin;
  int sel_above;
  int sel_count;
  int cnt;         // entries kept by compact_kept
  int pmax;        // highest kept position among keys tied at the cut
  __device__ uint32_t* bitmap() { return reinterpret_cast<uint32_t*>(&ring[0][0]); }
};

// Outcome of a radix select: keep key > thr, and the first keep_eq keys == thr
// in tie order; count_eq = how many input keys equal thr (when keep_eq > 0).
struct KeepRule {
  long long thr;
  int keep_eq;
  int count_eq;
};

// Bin (scanning from the top) where the running count of hist[0, NB) first
// reaches `need`; sets sel_bin, sel_above (count strictly above it) and
// sel_count.  Lane l of warp w holds NB / 1024 consecutive bins, warps and lanes
// ordered from the top; one warp scan finds the lane, which scans its own bins.
template <int NB>
__device__ void find_bin(int need, TopkShared& sh) {
  constexpr int kPerLane = NB / kTopkThreads;
  static_assert(kPerLane == 4 || kPerLane == 1, "bins per lane");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int lo = NB - (int(threadIdx.x) + 1) * kPerLane;  // this lane's lowest bin
  uint32_t c[kPerLane];
  if constexpr (kPerLane == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(&sh.hist[lo]);
    c[0] = v.x, c[1] = v.y, c[2] = v.z, c[3] = v.w;
  } else {
    c[0] = sh.hist[lo];
  }
  int s = 0;
#pragma unroll
  for (int q = 0; q < kPerLane; ++q) s += int(c[q]);
  const int inc = warp_inclusive_sum(s);
  const int wtot = __shfl_sync(0xffffffffu, inc, 31);
  if (lane == 0) sh.wsum[warp] = wtot;
  __syncthreads();
  const int winc = warp_inclusive_sum(int(sh.wsum[lane]));
  const int above = __shfl_sync(0xffffffffu, winc, (warp + 31) & 31) * (warp > 0);
  if (above < need && above + wtot >= need) {
    const unsigned hit = __ballot_sync(0xffffffffu, above + inc >= need);
    if (lane == __ffs(hit) - 1) {
      int run = above + inc - s;
#pragma unroll
      for (int q = kPerLane - 1; q >= 0; --q) {
        if (run + int(c[q]) >= need) {
          sh.sel_bin = lo + q;
          sh.sel_above = run;
          sh.sel_count = int(c[q]);
          break;
        }
        run += int(c[q]);
      }
    }
  }
  __syncthreads();
}

// Shared-memory histogram increment (plain atomics measured faster here than
// aggregating equal bins across a warp first).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) { atomicAdd(&hist[bin], 1u); }

template <int NB>
__device__ __forceinline__ void clear_hist(TopkShared& sh) {
  if constexpr (NB == kTopkThreads * 4)
    reinterpret_cast<uint4*>(sh.hist)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
  else
    for (int b = threadIdx.x; b < NB; b += kTopkThreads) sh.hist[b] = 0u;
}

// One radix pass: histogram of bits [shift, shift + log2 NB) of the keys whose
// bits above those equal `prefix`, then the bin holding the need-th largest.
template <int NB, class Key>
__device__ void radix_pass(int m, int need, uint32_t prefix, int bits_done, TopkShared& sh, Key key) {
  const int shift = 32 - bits_done - (NB == 4096 ? 12 : 10);
  clear_hist<NB>(sh);
  __syncthreads();
  for (int j = threadIdx.x; j < m; j += kTopkThreads) {
    const uint32_t k = key(j);
    if (bits_done == 0 || (k >> (32 - bits_done)) == prefix) hist_add(sh.hist, (k >> shift) & uint32_t(NB - 1));
  }
  __syncthreads();
  find_bin<NB>(need, sh);
}

// Radix selection of the `need`-th largest of m keys, 12 + 10 + 10 bits;
// key(j) reads key j.
template <class Key>
__device__ KeepRule radix_select(int m, int need, TopkShared& sh, Key key) {
  radix_pass<4096>(m, need, 0u, 0, sh, key);
  uint32_t prefix = uint32_t(sh.sel_bin);
  need -= sh.sel_above;
  if (sh.sel_count == need) return KeepRule{((long long)prefix << 20) - 1, 0, 0};  // whole bin kept
  radix_pass<1024>(m, need, prefix, 12, sh, key);
  prefix = (prefix << 10) | uint32_t(sh.sel_bin);
  need -= sh.sel_above;
  if (sh.sel_count == need) return KeepRule{((long long)prefix << 10) - 1, 0, 0};
  radix_pass<1024>(m, need, prefix, 22, sh, key);
  prefix = (prefix << 10) | uint32_t(sh.sel_bin);
  need -= sh.sel_above;
  if (sh.sel_count == need) return KeepRule{(long long)prefix - 1, 0, 0};
  return KeepRule{(long long)prefix, need, sh.sel_count};
}

// The kept set among the candidates: key > thr, or key == thr and the position
// passes the tie rule (the keep_eq lowest positions among the tied keys).
struct Selection {
  long long thr;
  int keep_eq;
  long long pthr;  // tie rule on ~pos: ~pos > pthr, or ~pos == pthr when pkeep > 0
  int pkeep;
  __device__ __forceinline__ bool kept(uint32_t key, int pos) const {
    if ((long long)key > thr) return true;
    if (keep_eq == 0 || (long long)key != thr) return false;
    const long long kp = (long long)(~uint32_t(pos));
    return kp > pthr || (kp == pthr && pkeep > 0);
  }
};

// Exact top-`topk` of the m >= topk candidates in the buffer.
__device__ Selection select_candidates(int m, int topk, TopkShared& sh) {
  const KeepRule r = radix_select(m, topk, sh, [&](int j) { return sh.cand_key[j]; });
  Selection s{r.thr, r.keep_eq, -1, 0};
  if (r.keep_eq > 0 && r.keep_eq < r.count_eq) {
    // only some of the tied keys fit: the keep_eq lowest positions, i.e. the
    // keep_eq largest ~pos (untied entries map to 0, below every ~pos)
    const uint32_t t = uint32_t(r.thr);
    const KeepRule p = radix_select(m, r.keep_eq, sh, [&](int j) {
      return sh.cand_key[j] == t ? ~uint32_t(sh.cand_pos[j]) : 0u;
    });
    s.pthr = p.thr;
    s.pkeep = p.keep_eq;
  }
  return s;
}

// Compacts the kept candidates of [0, m) to the front (any order); leaves their
// count in sh.cnt and the highest kept position tied at s.thr in sh.pmax.
__device__ void compact_kept(int m, const Selection& s, TopkShared& sh) {
  if (threadIdx.x == 0) {
    sh.cnt = 0;
    sh.pmax = -1;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int base = 0; base < m; base += kTopkThreads) {
    const int j = base + threadIdx.x;
    uint32_t key = 0;
    int pos = 0;
    bool keep = false;
    if (j < m) {
      key = sh.cand_key[j];
      pos = sh.cand_pos[j];
      keep = s.kept(key, pos);
    }
    // every entry of this round is in registers before any slot is written;
    // slots written now are < base + kTopkThreads, all of them read already
    __syncthreads();
    const unsigned bal = __ballot_sync(0xffffffffu, keep);
    int slot0 = 0;
    if (lane == 0 && bal) slot0 = atomicAdd(&sh.cnt, __popc(bal));
    slot0 = __shfl_sync(0xffffffffu, slot0, 0);
    if (keep) {
      const int o = slot0 + __popc(bal & ((1u << lane) - 1u));
      sh.cand_key[o] = key;
      sh.cand_pos[o] = pos;
      if (s.keep_eq > 0 && (long long)key == s.thr) atomicMax(&sh.pmax, pos);
    }
  }
  __syncthreads();
}

// Writes the kept candidates' positions in ascending order: per window of
// kBitmapWords * 32 positions, mark a bitmap (in the idle ring), scan its
// popcounts, emit.
__device__ void write_selected(int m, int n, const Selection& s, int topk, int32_t* __restrict__ out,
                               TopkShared& sh) {
  constexpr int kWin = kBitmapWords * 32;
  uint32_t* bitmap = sh.bitmap();
  int written = 0;
  for (int w0 = 0; w0 < n; w0 += kWin) {
    reinterpret_cast<uint4*>(bitmap)[threadIdx.x] = make_uint4(0u, 0u, 0u, 0u);
    __syncthreads();
    for (int j = threadIdx.x; j < m; j += kTopkThreads) {
      const int pos = sh.cand_pos[j];
      if (pos >= w0 && pos - w0 < kWin && s.kept(sh.cand_key[j], pos))
        atomicOr(&bitmap[(pos - w0) >> 5], 1u << (pos & 31));
    }
    __syncthreads();
    const uint4 a = reinterpret_cast<const uint4*>(bitmap)[threadIdx.x];
    const uint32_t wd[kWordsPerThread] = {a.x, a.y, a.z, a.w};
    int local = 0;
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) local += __popc(wd[q]);
    int tot = 0;
    int o = written + block_exclusive_sum<int>(local, sh.scan_i, &tot);
    const int pos0 = w0 + int(threadIdx.x) * kWordsPerThread * 32;
#pragma unroll
    for (int q = 0; q < kWordsPerThread; ++q) {
      uint32_t x = wd[q];
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        if (o < topk) out[o] = pos0 + q * 32 + bit;
        ++o;
      }
    }
    written += tot;
    // the scan's barriers separate every bitmap read above from the next clear
  }
  for (int j = written + int(threadIdx.x); j < topk; j += kTopkThreads) out[j] = -1;
}

// Ordered compaction of kept keys straight from global memory (the exact
// fallback).  get(j, key, pos) for j in [0, m), visited in position order.
template <class Get>
__device__ void write_kept(int m, KeepRule rule, int topk, int32_t* __restrict__ out, TopkShared& sh, Get get) {
  constexpr int kPer = 8;
  const int step = kTopkThreads * kPer;
  int written = 0, eq_seen = 0;
  for (int base = 0; base < m; base += step) {
    const int j0 = base + int(threadIdx.x) * kPer;
    int gt_mask = 0, eq_mask = 0;
    int pos[kPer];
#pragma unroll
    for (int t = 0; t < kPer; ++t) {
      pos[t] = -1;
      if (j0 + t < m) {
        uint32_t key;
        get(j0 + t, key, pos[t]);
        if ((long long)key > rule.thr) gt_mask |= 1 << t;
        else if ((long long)key == rule.thr) eq_mask |= 1 << t;
      }
    }
    int take_eq = 0, tot_e = 0;
    if (rule.keep_eq > 0) {
      int rnk = eq_seen + block_exclusive_sum<int>(__popc(eq_mask), sh.scan_i, &tot_e);
#pragma unroll
      for (int t = 0; t < kPer; ++t)
        if (eq_mask & (1 << t)) {
          if (rnk < rule.keep_eq) take_eq |= 1 << t;
          ++rnk;
        }
    }
    const int sel = gt_mask | take_eq;
    int tot_s = 0;
    int o = written + block_exclusive_sum<int>(__popc(sel), sh.scan_i, &tot_s);
#pragma unroll
    for (int t = 0; t < kPer; ++t)
      if (sel & (1 << t)) {
        if (o < topk) out[o] = pos[t];
        ++o;
      }
    written += tot_s;
    eq_seen += tot_e;
  }
  for (int j = written + int(threadIdx.x); j < topk; j += kTopkThreads) out[j] = -1;
}

// Moves every warp's region [reg_base, reg_base + wcnt) into one run starting
// at dst0, in warp order; returns dst0 + the total.  Each warp holds its entries
// in registers across a barrier, since a destination may overlap an earlier
// warp's region.
__device__ int gather_regions(int dst0, int reg_base, int wcnt, TopkShared& sh) {
  constexpr int kPerLane = (kCandCap / kTopkWarps + 31) / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t kk[kPerLane];
  int pp[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int j = lane + 32 * i;
    if (j < wcnt) {
      kk[i] = sh.cand_key[reg_base + j];
      pp[i] = sh.cand_pos[reg_base + j];
    }
  }
  if (lane == 0) sh.wsum[warp] = wcnt;
  __syncthreads();
  const int winc = warp_inclusive_sum(sh.wsum[lane]);
  const int total = __shfl_sync(0xffffffffu, winc, 31);
  const int dst = dst0 + __shfl_sync(0xffffffffu, winc, warp) - wcnt;
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const int j = lane + 32 * i;
    if (j < wcnt) {
      sh.cand_key[dst + j] = kk[i];
      sh.cand_pos[dst + j] = pp[i];
    }
  }
  __syncthreads();
  return dst0 + total;
}

// Threshold from a strided sample of kSamples keys: the lower edge of the 22-bit
// bin holding the rank-th largest sample key, so >= rank sample keys reach it.
__device__ uint32_t sample_threshold(const float* __restrict__ row, int n, int topk, TopkShared& sh) {
  const int stride = n / kSamples;  // >= 2 for rows longer than the buffer
  uint32_t key[kSamplesPerThread];
#pragma unroll
  for (int u = 0; u < kSamplesPerThread; ++u)
    key[u] = order_key(__ldg(row + (long long)(threadIdx.x + u * kTopkThreads) * stride));
  // expected share of the top-k in the sample, plus four standard deviations and slack
  const float share = float(topk) * float(kSamples) / float(n);
  const int rank = min(kSamples, int(ceilf(share + 4.0f * sqrtf(share))) + 8);
  clear_hist<4096>(sh);
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kSamplesPerThread; ++u) hist_add(sh.hist, key[u] >> 20);
  __syncthreads();
  find_bin<4096>(rank, sh);
  const uint32_t bin1 = uint32_t(sh.sel_bin);
  const int need = rank - sh.sel_above;
  clear_hist<1024>(sh);
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kSamplesPerThread; ++u)
    if ((key[u] >> 20) == bin1) hist_add(sh.hist, (key[u] >> 10) & 1023u);
  __syncthreads();
  find_bin<1024>(need, sh);
  return (bin1 << 20) | (uint32_t(sh.sel_bin) << 10);
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t score_ld,
                                                            const int32_t* __restrict__ n_vis, int topk,
                                                            int32_t* __restrict__ idx, int force_full, int split) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  pdl_wait();  // the scores come from the previous kernel
  pdl_trigger();
  // `split` CTAs (one cluster) per row; every branch below that returns early
  // depends on the row alone, so a cluster's CTAs take it together
  const int r = blockIdx.x / split;
  const int rank = split > 1 ? int(cluster_ctarank()) : 0;
  const int n = n_vis[r];
  int32_t* out = idx + (long long)r * topk;
  if (n < 1 || n > score_ld) {
    if (rank == 0 && threadIdx.x == 0) raise_status(kStatusBadRow);
    if (rank == 0)
      for (int j = threadIdx.x; j < topk; j += kTopkThreads) out[j] = -1;
    return;
  }
  if (n <= topk) {
    if (rank == 0)
      for (int j = threadIdx.x; j < topk; j += kTopkThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = scores + (long long)r * score_ld;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  const int nf4 = (n + 3) >> 2;  // float4s covering the row; the last may pass n, never score_ld

  int m = 0;
  if (force_full) {
    if (rank != 0) return;
  } else {
    if (n <= kCandCap) {
      if (rank != 0) return;
      // every key is a candidate, at its own position
      for (int f = threadIdx.x; f < nf4; f += kTopkThreads) {
        const float4 v = __ldg(row4 + f);
        const float x[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (4 * f + c < n) {
            sh.cand_key[4 * f + c] = order_key(x[c]);
            sh.cand_pos[4 * f + c] = 4 * f + c;
          }
      }
      __syncthreads();
      m = n;
    } else {
      // this CTA streams chunks [c_lo, c_lo + my_nch) of the row's nch
      const int nch = (nf4 + kChunkF4 - 1) / kChunkF4;
      const int per_rank = (nch + split - 1) / split;
      const int c_lo = min(nch, rank * per_rank);
      const int my_nch = min(nch, c_lo + per_rank) - c_lo;
      const uint32_t ring0 = smem_u32(&sh.ring[0][0]);
      auto issue = [&](int i) {
        if (i < my_nch) {
          const uint32_t dst = ring0 + uint32_t((i % kRing) * kChunkF4 + int(threadIdx.x)) * 16u;
#pragma unroll
          for (int u = 0; u < kChunkVec; ++u) {
            const int f = (c_lo + i) * kChunkF4 + u * kTopkThreads + int(threadIdx.x);
            if (f < nf4) cp_async_16(dst + uint32_t(u * kTopkThreads) * 16u, row4 + f, true);
          }
        }
        cp_async_commit();
      };
#pragma unroll
      for (int c = 0; c < kRing; ++c) issue(c);  // in flight while the sample is taken

      // accept x > Kf, or x == Kf at a position below P (P == INT_MAX: x >= Kf)
      float Kf = key_float(sample_threshold(row, n, topk, sh));
      int P = INT_MAX;
      const int warp = threadIdx.x >> 5;
      // Each warp appends to its own region of the buffer; [0, kept0) holds
      // the entries kept by the last cut.
      int kept0 = 0;
      int reg_cap = kCandCap / kTopkWarps;
      int reg_base = warp * reg_cap;
      int wcnt = 0;
      for (int i = 0; i < my_nch; ++i) {
        cp_async_wait_group<kRing - 1>();
        float x[kKeysPerThread];
#pragma unroll
        for (int u = 0; u < kChunkVec; ++u) {
          const float4 v = sh.ring[i % kRing][u * kTopkThreads + threadIdx.x];
          x[4 * u] = v.x, x[4 * u + 1] = v.y, x[4 * u + 2] = v.z, x[4 * u + 3] = v.w;
        }
        issue(i + kRing);  // refills this thread's own slots; the keys stay in registers
        const int f0 = (c_lo + i) * kChunkF4;
        const bool exact = (P != INT_MAX) || (c_lo + i == nch - 1);  // tie rule or ragged tail
        bool done = false;
        for (;;) {
          if (!done) {
            unsigned mine = 0u;
            if (!exact) {
#pragma unroll
              for (int t = 0; t < kKeysPerThread; ++t) mine |= unsigned(x[t] >= Kf) << t;
            } else {
#pragma unroll
              for (int t = 0; t < kKeysPerThread; ++t) {
                const int pos = 4 * (f0 + (t >> 2) * kTopkThreads + int(threadIdx.x)) + (t & 3);
                const bool pass = pos < n && (x[t] > Kf || (x[t] == Kf && pos < P));
                mine |= unsigned(pass) << t;
              }
            }
            const int cnt = __popc(mine);
            const int inc = warp_inclusive_sum(cnt);
            const int tot = __shfl_sync(0xffffffffu, inc, 31);
            if (wcnt + tot <= reg_cap) {
              int o = reg_base + wcnt + inc - cnt;
              while (mine) {
                const int t = __ffs(mine) - 1;
                mine &= mine - 1u;
                float v = x[0];
#pragma unroll
                for (int tt = 1; tt < kKeysPerThread; ++tt) v = (t == tt) ? x[tt] : v;
                sh.cand_key[o] = order_key(v);
                sh.cand_pos[o] = 4 * (f0 + (t >> 2) * kTopkThreads + int(threadIdx.x)) + (t & 3);
                ++o;
              }
              wcnt += tot;
              done = true;
            }
          }
          if (!__syncthreads_or(!done)) break;
          // A warp's region is full: gather the regions behind the kept run and,
          // with more than topk candidates, cut them to their exact top-k.
          const int m0 = gather_regions(kept0, reg_base, wcnt, sh);
          if (m0 > topk) {
            const Selection s = select_candidates(m0, topk, sh);
            compact_kept(m0, s, sh);
            if (s.keep_eq > 0) {
              Kf = key_float(uint32_t(s.thr));  // a real key: exact as a float
              P = sh.pmax;
            } else {
              Kf = key_float(uint32_t(s.thr + 1));  // every kept key is >= thr + 1
              P = INT_MAX;
            }
            kept0 = topk;
          } else {
            kept0 = m0;
          }
          reg_cap = (kCandCap - kept0) / kTopkWarps;  // >= 256: any warp's chunk fits
          reg_base = kept0 + warp * reg_cap;
          wcnt = 0;
        }
      }
      cp_async_wait_all();
      m = gather_regions(kept0, reg_base, wcnt, sh);
      if (split > 1) {
        // Rank 0 appends the other CTAs' lists through distributed shared memory
        // and selects once over the union.  Each CTA sends every key that passed
        // the shared threshold while its list fits its share of rank 0's buffer
        // (the usual case: about 1.4 k / split keys each); a longer list is cut
        // to its own exact top-k first (the union still holds the row's top-k).
        if (m > kCandCap / split) {
          const Selection s = select_candidates(m, topk, sh);
          compact_kept(m, s, sh);
          m = topk;
        }
        if (threadIdx.x == 0) sh.cnt = m;
        cluster_sync_all();
        if (rank == 0) {
          for (int q = 1; q < split; ++q) {
            const int mq = int(ld_shared_cluster_u32(map_shared_rank(smem_u32(&sh.cnt), uint32_t(q))));
            const uint32_t kq = map_shared_rank(smem_u32(&sh.cand_key[0]), uint32_t(q));
            const uint32_t pq = map_shared_rank(smem_u32(&sh.cand_pos[0]), uint32_t(q));
            for (int j = threadIdx.x; j < mq; j += kTopkThreads) {
              sh.cand_key[m + j] = ld_shared_cluster_u32(kq + 4u * uint32_t(j));
              sh.cand_pos[m + j] = int(ld_shared_cluster_u32(pq + 4u * uint32_t(j)));
            }
            m += mq;
          }
        }
        cluster_sync_all();  // the other CTAs' buffers stay alive until rank 0 has read them
        if (rank != 0) return;
      }
    }
  }

  if (m >= topk) {
    const Selection s = select_candidates(m, topk, sh);
    write_selected(m, n, s, topk, out, sh);
  } else {
    const KeepRule rule = radix_select(n, topk, sh, [&](int j) { return order_key(__ldg(row + j)); });
    write_kept(n, rule, topk, out, sh, [&](int j, uint32_t& key, int& pos) {
      key = order_key(__ldg(row + j));
      pos = j;
    });
  }
}

// Exact top-k of the candidate buffers a streamed indexer sweep leaves (one CTA
// per query row): the buffer's (key, position) pairs, in no particular order,
// are loaded into shared memory, selected (ties to lower positions) and written
// ascending through the position bitmap.  A row with cnt < 0 was never swept.
__global__ void __launch_bounds__(kTopkThreads) stream_select_kernel(const uint32_t* __restrict__ cand_key,
                                                                     const int32_t* __restrict__ cand_pos,
                                                                     const int* __restrict__ cnt, int cap,
                                                                     const int32_t* __restrict__ n_vis, int topk,
                                                                     int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int m = min(cnt[r], cap);
  if (m < 0) return;
  const long long ro = (long long)r * cap;
  for (int j = threadIdx.x; j < m; j += kTopkThreads) {
    sh.cand_key[j] = cand_key[ro + j];
    sh.cand_pos[j] = cand_pos[ro + j];
  }
  __syncthreads();
  Selection sel{-1, 0, -1, 0};  // fewer than topk candidates: keep them all
  if (m > topk) sel = select_candidates(m, topk, sh);
  write_selected(m, n_vis[r], sel, topk, idx + (long long)r * topk, sh);
}

}  // namespace

cudaError_t prepare_topk() {
  cudaError_t e =
      cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(TopkShared)));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(topk_short_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(ShortShared)));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(stream_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(sizeof(TopkShared)));
}

cudaError_t launch_stream_select(const StreamOut& so, const int32_t* n_vis, int T, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  static_assert(kStreamCap <= kCandCap, "a streamed candidate buffer fits the shared candidate arrays");
  return launch_pdl(stream_select_kernel, dim3(unsigned(T)), dim3(kTopkThreads), sizeof(TopkShared), stream, 1,
                    so.cand_key, so.cand_pos, so.cnt_out, so.cap, n_vis, so.topk, so.idx);
}

cudaError_t launch_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk, int32_t* idx,
                        int sm_count, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  // DSA_TOPK_KERNEL (tests): "row" skips the filter of the row kernel (its full
  // radix path), "short" takes the short-row kernel for any batch size
  const char* force = std::getenv("DSA_TOPK_KERNEL");
  const int force_full = (force && force[0] == 'r') ? 1 : 0;
  const bool force_short = force && force[0] == 's';
  // Many short rows: one row per 256-thread CTA, as many CTAs per SM as the kernel's launch bound allows.
  if (!force_full && score_ld <= kShortMaxN && (force_short || T >= 2 * sm_count))
    return launch_pdl(topk_short_kernel, dim3(unsigned(T)), dim3(kShortThreads), sizeof(ShortShared), stream, 1,
                      scores, score_ld, n_vis, topk, idx);
  // Few rows: split each long row over a cluster so more SMs stream it.
  int split = 1;
  if (const char* sp = std::getenv("DSA_TOPK_SPLIT")) {  // tests pin 1, 2 or 4
    split = std::atoi(sp);
  } else if (score_ld >= int64_t(4) * kChunkF4 * 4 && sm_count >= 2 * T) {
    split = sm_count / T;
  }
  split = split >= 4 ? 4 : (split >= 2 ? 2 : 1);
  static_assert(4 * DSA_MAX_TOPK <= kCandCap, "rank 0 holds every CTA's list (at most max(topk, kCandCap / split))");
  return launch_pdl(topk_kernel, dim3(unsigned(T) * unsigned(split)), dim3(kTopkThreads), sizeof(TopkShared), stream,
                    unsigned(split), scores, score_ld, n_vis, topk, idx, force_full, split);
}

}  // namespace dsa
