// Exact per-row top-k for batches of short rows (at most kShortMaxN scores),
// such as the rows of a causal prefill.
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.2: keep the index_topk highest-scoring positions.  Ties go to the
// lower position; the kept positions are written in ascending order and padded
// with -1.)
//
// The row kernel of topk.cuh gives each row a 1024-thread CTA that fills an SM;
// on a row of a few thousand scores its phases are short and separated by
// block-wide barriers, so the SM mostly waits.  Here a row gets a 256-thread
// CTA of 41 KB and 48 registers a thread, five rows share an SM and one row's
// barrier waits overlap another's work.  Per row:
//   1. a row longer than the candidate buffer takes a strided sample of 1024
//      keys and selects its rank-th largest, rank a few standard deviations
//      above the sample's expected share of k: keys above that threshold t are
//      candidates (a shorter row keeps every key);
//   2. one pass over the row appends the candidates, with their positions, to
//      the buffer (warp scan, one shared atomic per warp);
//   3. if at least k keys passed and they fit, the exact radix select of
//      group_select.cuh runs over the buffer (a second select over positions
//      when only some keys tied at the k-th place fit) -- every key tied with
//      the k-th is above t, so the candidates hold the row's top-k; otherwise
//      the same select runs over the row in global memory.  The candidates'
//      keys are first mapped onto the full 32 bits (minus t + 1, shifted left
//      by the range's leading zeros: order-preserving and one-to-one), and the
//      digits are four 8-bit passes, so the histogram a pass clears and scans
//      is 256 bins (one per thread) -- the shared-memory pipe, not the data,
//      set this kernel's pace with 4096-bin passes;
//   4. the kept positions are marked in a bitmap of the row and written in
//      ascending order after a block scan of the words' popcounts.
#pragma once
#include <cuda_runtime.h>

#include "block_scan.cuh"
#include "dsa.h"
#include "group_select.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kShortThreads = 256;
constexpr int kShortMaxN = 32768;                       // longest row this kernel takes
constexpr int kShortCap = 4608;                         // candidate entries (about 4 sigma above a 32K row's expectation)
constexpr int kShortSamples = 4 * kShortThreads;        // 1024
constexpr int kShortBitmapWords = kShortMaxN / 32;      // one bit per position
constexpr int kShortWordsPerThread = kShortBitmapWords / kShortThreads;
constexpr int kShortVec = 2;                            // float4 loads in flight per thread
constexpr int kShortSub = 2;                            // float4s filtered at a time
static_assert(kShortCap >= kShortSamples, "the sample sits in the candidate keys");
static_assert(kShortCap > DSA_MAX_TOPK, "the buffer holds more than k candidates");

// Radix digits of the selections: four 8-bit passes, so each pass clears and
// scans a 256-bin histogram (one bin per thread) instead of 4096 bins.
constexpr int kShortBins = 256;
__device__ constexpr int kShortDigits[4] = {8, 8, 8, 8};  // 1 << 8 == kShortBins

struct ShortShared {
  uint32_t cand_key[kShortCap];
  int32_t cand_pos[kShortCap];
  uint32_t hist[kShortBins];
  uint32_t bitmap[kShortBitmapWords];
  GroupShared gs;
  int cnt;
  uint32_t kmax;  // largest candidate key
};

__device__ __forceinline__ uint32_t short_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kShortThreads, 5)
    topk_short_kernel(const float* __restrict__ scores, int64_t score_ld, const int32_t* __restrict__ n_vis, int topk,
                      int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t short_smem[];
  ShortShared& sh = *reinterpret_cast<ShortShared*>(short_smem);
  pdl_wait();  // the scores come from the previous kernel
  pdl_trigger();
  const int r = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int n = n_vis[r];
  int32_t* out = idx + (long long)r * topk;
  if (n < 1 || n > score_ld || n > kShortMaxN) {
    if (tid == 0) raise_status(kStatusBadRow);
    for (int j = tid; j < topk; j += kShortThreads) out[j] = -1;
    return;
  }
  if (n <= topk) {
    for (int j = tid; j < topk; j += kShortThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* row = scores + (long long)r * score_ld;
  const Group g{tid, kShortThreads, 1};

  // 1. candidate threshold: a key passes when key > t
  long long t = -1;
  if (n > kShortCap) {
    const int stride = n / kShortSamples;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = tid + u * kShortThreads;
      sh.cand_key[j] = short_order_key(__ldg(row + (long long)j * stride));
    }
    g.sync();
    const float share = float(topk) * float(kShortSamples) / float(n);
    const int rank = min(kShortSamples, int(ceilf(share + 4.0f * sqrtf(share))) + 8);
    const Rule rs = group_radix_select_digits(kShortSamples, rank, sh.hist, sh.gs, g,
                                              [&](int j) { return sh.cand_key[j]; }, [](int) { return true; },
                                              kShortDigits, 4);
    t = rs.keep_eq > 0 ? rs.thr - 1 : rs.thr;  // at least `rank` sample keys are above t
  }
  if (tid == 0) {
    sh.cnt = 0;
    sh.kmax = 0u;
  }
  g.sync();  // the sample is consumed and the count cleared before any append
  uint32_t my_max = 0u;

  // 2. one pass: append the keys above t with their positions
  const float4* row4 = reinterpret_cast<const float4*>(row);
  const int nf4 = (n + 3) >> 2;  // the last float4 may pass n, never score_ld
  for (int f0 = 0; f0 < nf4; f0 += kShortThreads * kShortVec) {
    float4 v[kShortVec];
#pragma unroll
    for (int u = 0; u < kShortVec; ++u) {
      const int f = f0 + u * kShortThreads + tid;
      if (f < nf4) v[u] = __ldg(row4 + f);
    }
#pragma unroll
    for (int s0 = 0; s0 < kShortVec; s0 += kShortSub) {
      uint32_t key[4 * kShortSub];
      uint32_t mask = 0u;
#pragma unroll
      for (int u = 0; u < kShortSub; ++u) {
        const int f = f0 + (s0 + u) * kShortThreads + tid;
        const float x[4] = {v[s0 + u].x, v[s0 + u].y, v[s0 + u].z, v[s0 + u].w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          key[4 * u + c] = short_order_key(x[c]);
          const bool pass = f < nf4 && 4 * f + c < n && (long long)key[4 * u + c] > t;
          mask |= uint32_t(pass) << (4 * u + c);
        }
      }
      const int cnt = __popc(mask);
      const int inc = warp_inclusive_sum(cnt);
      int base = 0;
      if (lane == 31 && inc > 0) base = atomicAdd(&sh.cnt, inc);
      base = __shfl_sync(0xffffffffu, base, 31);
      int o = base + inc - cnt;
#pragma unroll
      for (int b = 0; b < 4 * kShortSub; ++b)
        if ((mask >> b) & 1u) {
          if (o < kShortCap) {
            sh.cand_key[o] = key[b];
            sh.cand_pos[o] = 4 * (f0 + (s0 + (b >> 2)) * kShortThreads + tid) + (b & 3);
          }
          my_max = key[b] > my_max ? key[b] : my_max;
          ++o;
        }
    }
  }
  if (my_max) atomicMax(&sh.kmax, my_max);
  g.sync();
  const int passed = sh.cnt;

  // 3. exact selection over the candidates, or over the row when the filter
  //    let fewer than k keys through (a sample far off its expectation) or
  //    more than the buffer holds; 4. ordered output through the bitmap
  auto finish = [&](int m, auto key_of, auto pos_of) {
    const Rule rr =
        group_radix_select_digits(m, topk, sh.hist, sh.gs, g, key_of, [](int) { return true; }, kShortDigits, 4);
    long long cut = 0;  // among keys == rr.thr keep positions p with ~p >= cut
    if (rr.keep_eq > 0 && rr.keep_eq < rr.count_eq) {  // only the lowest tied positions fit
      const Rule rp = group_radix_select_digits(
          m, rr.keep_eq, sh.hist, sh.gs, g, [&](int j) { return ~uint32_t(pos_of(j)); },
          [&](int j) { return (long long)key_of(j) == rr.thr; }, kShortDigits, 4);
      cut = rp.keep_eq > 0 ? rp.thr : rp.thr + 1;
    }
    for (int w = tid; w < kShortBitmapWords; w += kShortThreads) sh.bitmap[w] = 0u;
    g.sync();
    for (int j = tid; j < m; j += kShortThreads) {
      const long long k = key_of(j);
      const int p = pos_of(j);
      if (k > rr.thr || (rr.keep_eq > 0 && k == rr.thr && (long long)(~uint32_t(p)) >= cut))
        atomicOr(&sh.bitmap[p >> 5], 1u << (p & 31));
    }
    g.sync();
    uint32_t wd[kShortWordsPerThread];
    int local = 0;
#pragma unroll
    for (int q = 0; q < kShortWordsPerThread; ++q) {
      wd[q] = sh.bitmap[tid * kShortWordsPerThread + q];
      local += __popc(wd[q]);
    }
    int total = 0;
    int o = group_exclusive_sum(local, sh.gs, &total, g);
#pragma unroll
    for (int q = 0; q < kShortWordsPerThread; ++q) {
      uint32_t x = wd[q];
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        if (o < topk) out[o] = (tid * kShortWordsPerThread + q) * 32 + bit;
        ++o;
      }
    }
    for (int j = total + tid; j < topk; j += kShortThreads) out[j] = -1;
  };
  if (passed >= topk && passed <= kShortCap) {
    // Every candidate key lies in (t, kmax]: select on (key - t - 1) << z, z the
    // leading zeros of that range, an order-preserving one-to-one map that
    // spreads the candidates over the first radix pass's bins (raw keys of the
    // top few percent of a row share most of their top 12 bits, and the
    // histogram atomics would pile into a few dozen bins).
    const uint32_t lo = uint32_t(t + 1);
    const uint32_t span = sh.kmax - lo;
    const int z = span ? __clz(span) : 0;
    finish(passed, [&](int j) { return (sh.cand_key[j] - lo) << z; }, [&](int j) { return sh.cand_pos[j]; });
  } else
    finish(n, [&](int j) { return short_order_key(__ldg(row + j)); }, [](int j) { return j; });
}

}  // namespace

}  // namespace dsa
