// Exact per-row top-k over materialised fp32 indexer scores.
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.2: keep the index_topk highest-scoring positions.  Ties go to the
// lower position; the kept positions are written in ascending order and padded
// with -1.)
//
// Scores map to 32-bit keys whose unsigned order is the float order (-0 is
// folded onto +0), so "k-th largest" is a radix select on keys.  One CTA per
// row:
//   1. rows longer than the candidate buffer first take a strided sample of
//      kSamples keys; the r-th largest sample key, r about twice the sample's
//      share of k, is a threshold tau_lo that at least k and at most a few
//      thousand of the row's keys reach, with overwhelming probability;
//   2. one streaming pass (deep loads, ordered compaction with block scans)
//      copies every key >= tau_lo and its position into shared memory, in
//      position order;
//   3. an exact radix select over those candidates (12 + 10 + 10 bit
//      histograms in shared memory) gives the k-th key tau and how many keys
//      equal to tau are kept, and a final ordered compaction writes the kept
//      positions: ascending, ties to the lowest positions.
// Steps 1-2 are a filter, not an approximation: if fewer than k keys reach
// tau_lo, or more than the buffer holds, the row is redone by the full
// multi-pass radix select over global memory, which is always exact.
#pragma once
#include <cstdlib>

#include "block_scan.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kSamples = 4096;
constexpr int kCandCap = 8192;
constexpr int kHistBins = 4096;

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkShared {
  uint32_t hist[kHistBins];
  uint32_t samp[kSamples];
  uint32_t cand_key[kCandCap];
  int32_t cand_pos[kCandCap];
  int scan_i[33];
  int sel_bin;
  int sel_above;
  int sel_count;
};

// Keep rule of a finished selection: key > thr, or key == thr for the first
// keep_eq such keys in position order.
struct KeepRule {
  long long thr;
  int keep_eq;
};

// Bin b (scanning from the top) where the running count first reaches `need`.
__device__ void find_bin(int nb, int need, TopkShared& sh) {
  const int per = nb / int(blockDim.x) > 0 ? nb / int(blockDim.x) : 1;
  int local = 0;
  const int top = nb - 1 - int(threadIdx.x) * per;
  const bool owns = int(threadIdx.x) * per < nb;
  if (owns)
    for (int q = 0; q < per; ++q) local += int(sh.hist[top - q]);
  int total = 0;
  const int ex = block_exclusive_sum<int>(local, sh.scan_i, &total);
  if (owns && ex < need && ex + local >= need) {
    int run = ex;
    for (int q = 0; q < per; ++q) {
      const int c = int(sh.hist[top - q]);
      if (run + c >= need) {
        sh.sel_bin = top - q;
        sh.sel_above = run;
        sh.sel_count = c;
        break;
      }
      run += c;
    }
  }
  __syncthreads();
}

// Add 1 to hist[bin] for every calling lane; lanes of a warp with equal bins add
// once (candidate keys crowd into a few bins, where plain atomics serialise).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin) {
  const unsigned mask = __activemask();
  const unsigned peers = __match_any_sync(mask, bin);
  if ((threadIdx.x & 31) == unsigned(__ffs(peers) - 1)) atomicAdd(&hist[bin], uint32_t(__popc(peers)));
}

// Radix selection of the `need`-th largest of m keys, 12 + 10 + 10 bits;
// key(j) reads key j.
template <class Key>
__device__ KeepRule radix_select(int m, int need, TopkShared& sh, Key key) {
  uint32_t prefix = 0;
  int bits_done = 0;
  const int widths[3] = {12, 10, 10};
  for (int p = 0; p < 3; ++p) {
    const int w = widths[p];
    const int shift = 32 - bits_done - w;
    const int nb = 1 << w;
    for (int b = threadIdx.x; b < nb; b += blockDim.x) sh.hist[b] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < m; j += blockDim.x) {
      const uint32_t k = key(j);
      if (bits_done == 0 || (k >> (32 - bits_done)) == prefix) hist_add(sh.hist, (k >> shift) & uint32_t(nb - 1));
    }
    __syncthreads();
    find_bin(nb, need, sh);
    prefix = (prefix << w) | uint32_t(sh.sel_bin);
    need -= sh.sel_above;
    bits_done += w;
    const bool whole = (sh.sel_count == need);
    __syncthreads();
    if (whole) return KeepRule{((long long)prefix << (32 - bits_done)) - 1, 0};  // the whole bin is kept
  }
  return KeepRule{(long long)prefix, need};
}

// Ordered compaction of kept keys.  get(j, key, pos) for j in [0, m), visited in
// position order; writes out[0:topk).
template <class Get>
__device__ void write_kept(int m, KeepRule rule, int topk, int32_t* __restrict__ out, TopkShared& sh, Get get) {
  constexpr int kPer = 8;
  const int step = int(blockDim.x) * kPer;
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
  for (int j = written + int(threadIdx.x); j < topk; j += blockDim.x) out[j] = -1;
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t score_ld,
                                                            const int32_t* __restrict__ n_vis, int topk,
                                                            int32_t* __restrict__ idx, int force_full) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(topk_smem);
  const int r = blockIdx.x;
  const int n = n_vis[r];
  int32_t* out = idx + (long long)r * topk;
  if (n < 1 || n > score_ld) {
    if (threadIdx.x == 0) raise_status(kStatusBadRow);
    for (int j = threadIdx.x; j < topk; j += blockDim.x) out[j] = -1;
    return;
  }
  if (n <= topk) {
    for (int j = threadIdx.x; j < topk; j += blockDim.x) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = scores + (long long)r * score_ld;

  bool filtered = false;
  int m = 0;  // candidates in shared memory
  if (!force_full) {
    // ---- threshold tau_lo: every key when the row fits the buffer, else from a strided sample
    uint32_t tau_lo = 0u;
    if (n > kCandCap) {
      const int stride = n / kSamples;
      for (int i = threadIdx.x; i < kSamples; i += blockDim.x)
        sh.samp[i] = order_key(__ldg(row + (long long)i * stride));
      __syncthreads();
      // the sample holds about topk * kSamples / n of the row's top-k keys; take twice that, plus slack
      const long long share = ((long long)topk * kSamples + n - 1) / n;
      const int rank = int(min(2 * share + 32, (long long)kSamples));
      const KeepRule s = radix_select(kSamples, rank, sh, [&](int j) { return sh.samp[j]; });
      tau_lo = uint32_t(s.keep_eq > 0 ? s.thr : s.thr + 1);  // the rank-th largest sample key, or below it
    }
    // ---- one streaming pass: candidates (key >= tau_lo) in position order
    constexpr int kVec = 8;  // float4 loads in flight per thread
    const int per_iter = int(blockDim.x) * kVec * 4;
    const int n_main = (n / per_iter) * per_iter;
    int total = 0;
    // the next iteration's loads are issued before this one is compacted
    float4 nxt[kVec];
    if (n_main > 0) {
      const float4* p4 = reinterpret_cast<const float4*>(row + int(threadIdx.x) * kVec * 4);
#pragma unroll
      for (int u = 0; u < kVec; ++u) nxt[u] = __ldg(p4 + u);
    }
    for (int base = 0; base < n; base += per_iter) {
      uint32_t keys[kVec * 4];
      const int j0 = base + int(threadIdx.x) * kVec * 4;  // this thread's 32 consecutive positions
      if (base < n_main) {
        float4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) v[u] = nxt[u];
        if (base + per_iter < n_main) {
          const float4* p4 = reinterpret_cast<const float4*>(row + j0 + per_iter);
#pragma unroll
          for (int u = 0; u < kVec; ++u) nxt[u] = __ldg(p4 + u);
        }
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
          keys[4 * u] = order_key(v[u].x);
          keys[4 * u + 1] = order_key(v[u].y);
          keys[4 * u + 2] = order_key(v[u].z);
          keys[4 * u + 3] = order_key(v[u].w);
        }
      } else {
#pragma unroll
        for (int t = 0; t < kVec * 4; ++t) keys[t] = (j0 + t < n) ? order_key(__ldg(row + j0 + t)) : 0u;
      }
      unsigned sel = 0u;
#pragma unroll
      for (int t = 0; t < kVec * 4; ++t)
        if (j0 + t < n && keys[t] >= tau_lo) sel |= 1u << t;
      int tot = 0;
      int o = total + block_exclusive_sum<int>(__popc(sel), sh.scan_i, &tot);
#pragma unroll
      for (int t = 0; t < kVec * 4; ++t)
        if (sel & (1u << t)) {
          if (o < kCandCap) {
            sh.cand_key[o] = keys[t];
            sh.cand_pos[o] = j0 + t;
          }
          ++o;
        }
      total += tot;
    }
    __syncthreads();
    filtered = (total >= topk && total <= kCandCap);
    m = total;
  }

  if (filtered) {
    const KeepRule rule = radix_select(m, topk, sh, [&](int j) { return sh.cand_key[j]; });
    write_kept(m, rule, topk, out, sh, [&](int j, uint32_t& key, int& pos) {
      key = sh.cand_key[j];
      pos = sh.cand_pos[j];
    });
  } else {
    const KeepRule rule = radix_select(n, topk, sh, [&](int j) { return order_key(__ldg(row + j)); });
    write_kept(n, rule, topk, out, sh, [&](int j, uint32_t& key, int& pos) {
      key = order_key(__ldg(row + j));
      pos = j;
    });
  }
}

}  // namespace

cudaError_t prepare_topk() {
  return cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sizeof(TopkShared)));
}

cudaError_t launch_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk, int32_t* idx,
                        cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const char* force = std::getenv("DSA_TOPK_KERNEL");  // "row": skip the filter (tests of the full path)
  const int force_full = (force && force[0] == 'r') ? 1 : 0;
  topk_kernel<<<T, kTopkThreads, sizeof(TopkShared), stream>>>(scores, score_ld, n_vis, topk, idx, force_full);
  return cudaGetLastError();
}

}  // namespace dsa
