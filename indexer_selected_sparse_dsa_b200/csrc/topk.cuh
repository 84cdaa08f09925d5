// Exact per-row top-k over materialised fp32 indexer scores.
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2: keep the index_topk
// highest-scoring positions; ties go to the lower position, the kept
// positions are written in ascending order and padded with -1.)
//
// One CTA per row.  Scores map to 32-bit keys whose unsigned order is the
// float order (-0 folded onto +0).  Three histogram passes (12 + 12 + 8 bits)
// find the k-th largest key tau and how many of the keys equal to tau are
// kept; a final pass compacts the kept positions in position order with
// block-wide scans, so the output is ascending by construction and ties at
// tau go to the lowest positions.
#pragma once
#include "block_scan.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kTopkThreads = 512;
constexpr int kBins = 4096;

__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;  // -0.0 == +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct TopkShared {
  unsigned int hist[kBins];
  long long scan_l[33];
  int scan_i[33];
  int sel_bin;
  int sel_above;  // count strictly above the selected bin
};

// Histogram pass over the row: bins of `bits` bits starting at bit `shift`,
// restricted to keys whose bits above (shift + bits) equal `prefix`.
__device__ void histogram_pass(const float* __restrict__ row, int n, int shift, int bits, uint32_t prefix,
                               TopkShared& sh) {
  const int nb = 1 << bits;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) sh.hist[b] = 0u;
  __syncthreads();
  const int hi_shift = shift + bits;
  const uint32_t mask = uint32_t(nb - 1);
  const int n4 = n >> 2;
  const float4* row4 = reinterpret_cast<const float4*>(row);
  for (int j = threadIdx.x; j < n4; j += blockDim.x) {
    float4 v = __ldg(row4 + j);
    float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t k = order_key(e[t]);
      if (hi_shift >= 32 || (k >> hi_shift) == prefix) atomicAdd(&sh.hist[(k >> shift) & mask], 1u);
    }
  }
  for (int j = (n4 << 2) + threadIdx.x; j < n; j += blockDim.x) {
    uint32_t k = order_key(__ldg(row + j));
    if (hi_shift >= 32 || (k >> hi_shift) == prefix) atomicAdd(&sh.hist[(k >> shift) & mask], 1u);
  }
  __syncthreads();
}

// Find the bin b (scanning from the top) where the running count first reaches
// `need`; returns in sh.sel_bin / sh.sel_above.
__device__ void find_bin(int bits, int need, TopkShared& sh) {
  const int nb = 1 << bits;
  const int per = nb / blockDim.x > 0 ? nb / blockDim.x : 1;
  // thread t owns bins [hi - per*(t+1) + 1, hi - per*t] counted from the top
  int local = 0;
  const int top = nb - 1 - int(threadIdx.x) * per;
  if (int(threadIdx.x) * per < nb)
    for (int q = 0; q < per; ++q) local += int(sh.hist[top - q]);
  int total = 0;
  int ex = block_exclusive_sum<int>(local, sh.scan_i, &total);
  if (int(threadIdx.x) * per < nb && ex < need && ex + local >= need) {
    int run = ex;
    for (int q = 0; q < per; ++q) {
      const int b = top - q;
      const int c = int(sh.hist[b]);
      if (run + c >= need) {
        sh.sel_bin = b;
        sh.sel_above = run;
        break;
      }
      run += c;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t score_ld,
                                                            const int32_t* __restrict__ n_vis, int topk,
                                                            int32_t* __restrict__ idx) {
  __shared__ TopkShared sh;
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

  // ---- radix passes: find tau (exact k-th largest key) and how many ties to keep
  int need = topk;
  uint32_t prefix = 0;
  const int shifts[3] = {20, 8, 0};
  const int widths[3] = {12, 12, 8};
  bool whole_bin = false;
  int bits_done = 0;
  for (int p = 0; p < 3; ++p) {
    histogram_pass(row, n, shifts[p], widths[p], prefix, sh);
    find_bin(widths[p], need, sh);
    const int b = sh.sel_bin;
    need -= sh.sel_above;
    prefix = (prefix << widths[p]) | uint32_t(b);
    bits_done += widths[p];
    if (int(sh.hist[b]) == need) {  // the whole bin is kept: no finer split needed
      whole_bin = true;
      break;
    }
    __syncthreads();
  }
  // Keep rule: key > thr, or key == thr for the first `keep_eq` such positions.
  // A whole kept bin is expressed as key >= lo (thr = lo - 1, keep_eq = 0).
  long long thr;
  int keep_eq;
  if (whole_bin) {
    const long long lo = (long long)prefix << (32 - bits_done);
    thr = lo - 1;
    keep_eq = 0;
  } else {
    thr = (long long)prefix;
    keep_eq = need;
  }

  // ---- ordered compaction: position order == ascending output
  const int per_thread = 4;
  const int chunk = kTopkThreads * per_thread;
  int written = 0, eq_seen = 0;
  for (int base = 0; base < n; base += chunk) {
    const int j0 = base + threadIdx.x * per_thread;
    int gt_mask = 0, eq_mask = 0;
#pragma unroll
    for (int t = 0; t < per_thread; ++t) {
      const int j = j0 + t;
      if (j < n) {
        const long long k = (long long)order_key(__ldg(row + j));
        if (k > thr) gt_mask |= 1 << t;
        else if (k == thr) eq_mask |= 1 << t;
      }
    }
    int tot_eq = 0;
    const int ex_eq = block_exclusive_sum<int>(__popc(eq_mask), sh.scan_i, &tot_eq);
    int take_eq = 0;
    int rank = eq_seen + ex_eq;
#pragma unroll
    for (int t = 0; t < per_thread; ++t)
      if (eq_mask & (1 << t)) {
        if (rank < keep_eq) take_eq |= 1 << t;
        ++rank;
      }
    const int sel_mask = gt_mask | take_eq;
    int tot_sel = 0;
    const int ex_sel = block_exclusive_sum<int>(__popc(sel_mask), sh.scan_i, &tot_sel);
    int pos = written + ex_sel;
#pragma unroll
    for (int t = 0; t < per_thread; ++t)
      if (sel_mask & (1 << t)) {
        if (pos < topk) out[pos] = j0 + t;
        ++pos;
      }
    written += tot_sel;
    eq_seen += tot_eq;
  }
  for (int j = written + threadIdx.x; j < topk; j += blockDim.x) out[j] = -1;
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk, int32_t* idx,
                        cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  topk_kernel<<<T, kTopkThreads, 0, stream>>>(scores, score_ld, n_vis, topk, idx);
  return cudaGetLastError();
}

}  // namespace dsa
