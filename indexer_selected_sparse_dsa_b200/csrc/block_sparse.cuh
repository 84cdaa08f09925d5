// Block-level variant: three branches over 128-token blocks, fused per head.
//
// ("GLM-5: 744B parameters, 202K long context", section 2, "Decoupled Sparse
// Attention": the context is cut into 128-token blocks; a local branch attends
// the query's block and its neighbours (O(N * 384)), a global anchor branch one
// block in every 16, and a dynamic branch each query's 16 most relevant blocks;
// the three outputs are fused with learned weights.)  The page does not say how
// a block is scored; here its score is the largest lightning-indexer score
// among its visible positions, and the 16 best blocks are kept under (score
// descending, block ascending) by the exact top-k kernel.  Each branch is the
// sparse MLA kernel over the branch's index list; the fusion weights are the
// caller's, per (row, head, branch).
//
//   block_max_kernel     scores [T, score_ld] -> block scores [T, bld], block counts [T]
//   (top-k kernel, k = 16)                   -> dynamic blocks [T, 16], ascending
//   block_expand_kernel  blocks, n_vis       -> index lists: local [T, 384],
//                                               anchor [T, wa], dynamic [T, 2048]
//   (sparse MLA kernel x 3)
//   fuse3_kernel         o = g_dyn o + g_local o_local + g_anchor o_anchor
#pragma once
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kBlockWarps = 8;  // one 128-position block per warp

// bscore[i, b] = max of scores[i, s] over block b's visible positions
// s in [128 b, min(128 b + 128, n_vis[i])); nblocks[i] = ceil(n_vis[i] / 128).
// Grid (ceil(max blocks / 8), T); rows with n_vis out of [1, score_ld] get 0 blocks
// (and a status bit).
__global__ void __launch_bounds__(32 * kBlockWarps) block_max_kernel(const float* __restrict__ scores,
                                                                     int64_t score_ld,
                                                                     const int32_t* __restrict__ n_vis, int bld,
                                                                     float* __restrict__ bscore,
                                                                     int32_t* __restrict__ nblocks) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.y;
  const int n = n_vis[i];
  const bool row_ok = n >= 1 && n <= score_ld && (n + kBlockTokens - 1) / kBlockTokens <= bld;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    nblocks[i] = row_ok ? (n + kBlockTokens - 1) / kBlockTokens : 0;
    if (!row_ok) raise_status(kStatusBadRow);
  }
  if (!row_ok) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x * kBlockWarps + warp;
  if (b * kBlockTokens >= n) return;
  const float* row = scores + (long long)i * score_ld + (long long)b * kBlockTokens;
  const int nb = min(kBlockTokens, n - b * kBlockTokens);  // visible positions of this block
  float m = -INFINITY;
#pragma unroll
  for (int u = 0; u < kBlockTokens / 32; ++u) {
    const int s = u * 32 + lane;
    if (s < nb) m = fmaxf(m, row[s]);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  if (lane == 0) bscore[(long long)i * bld + b] = m;
}

// The three index lists of row i (positions relative to kv_start, -1 = empty):
//   local:   max(0, 128 (qb - 1)) .. t, qb = t / 128 the query's block (the later
//            neighbour is in the future), padded to 384;
//   anchor:  the visible positions of blocks 0, 16, 32, ... <= qb, block by block;
//   dynamic: the visible positions of the row's selected blocks, block by block.
// All ascending.
__global__ void block_expand_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ n_vis,
                                    int wa, int32_t* __restrict__ idx_loc, int32_t* __restrict__ idx_anc,
                                    int32_t* __restrict__ idx_dyn) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  const int n = n_vis[i];
  const int t = n - 1;  // n < 1: every list empty
  const int qb = t >= 0 ? t / kBlockTokens : -1;
  int32_t* loc = idx_loc + (long long)i * kLocalWidth;
  int32_t* anc = idx_anc + (long long)i * wa;
  int32_t* dyn = idx_dyn + (long long)i * kDynWidth;
  const int lo = max(0, (qb - 1) * kBlockTokens);
  for (int e = threadIdx.x; e < kLocalWidth; e += blockDim.x) {
    const int p = lo + e;
    loc[e] = (t >= 0 && p <= t) ? p : -1;
  }
  for (int e = threadIdx.x; e < wa; e += blockDim.x) {
    const int b = (e / kBlockTokens) * kAnchorEvery;
    const int p = b * kBlockTokens + e % kBlockTokens;
    anc[e] = (b <= qb && p <= t) ? p : -1;
  }
  const int32_t* bl = blocks + (long long)i * kBlockTopk;
  for (int e = threadIdx.x; e < kDynWidth; e += blockDim.x) {
    const int b = bl[e / kBlockTokens];
    const int p = b * kBlockTokens + e % kBlockTokens;
    dyn[e] = (b >= 0 && p <= t) ? p : -1;
  }
}

// o = g_dyn * o + g_local * o_loc + g_anchor * o_anc, gates [T, 64, 3] = (local, anchor, dynamic).
__global__ void fuse3_kernel(float* __restrict__ o, const float* __restrict__ o_loc, const float* __restrict__ o_anc,
                             const float* __restrict__ gates, long long n4) {
  pdl_wait();
  pdl_trigger();
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n4; v += (long long)gridDim.x * blockDim.x) {
    const float* g = gates + ((v * 4) >> 9) * 3;  // 512 latent dims per (row, head)
    const float gl = g[0], ga = g[1], gd = g[2];
    const float4 a = reinterpret_cast<const float4*>(o_loc)[v];
    const float4 c = reinterpret_cast<const float4*>(o_anc)[v];
    float4 d = reinterpret_cast<float4*>(o)[v];
    d.x = gd * d.x + gl * a.x + ga * c.x;
    d.y = gd * d.y + gl * a.y + ga * c.y;
    d.z = gd * d.z + gl * a.z + ga * c.z;
    d.w = gd * d.w + gl * a.w + ga * c.w;
    reinterpret_cast<float4*>(o)[v] = d;
  }
}

}  // namespace

cudaError_t launch_block_max(const float* scores, int64_t score_ld, const int32_t* n_vis, int T, int bld,
                             float* bscore, int32_t* nblocks, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const dim3 grid(unsigned((bld + kBlockWarps - 1) / kBlockWarps), unsigned(T));
  return launch_pdl(block_max_kernel, grid, dim3(32 * kBlockWarps), 0, stream, 1, scores, score_ld, n_vis, bld,
                    bscore, nblocks);
}

cudaError_t launch_block_expand(const int32_t* blocks, const int32_t* n_vis, int T, int wa, int32_t* idx_loc,
                                int32_t* idx_anc, int32_t* idx_dyn, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl(block_expand_kernel, dim3(unsigned(T)), dim3(256), 0, stream, 1, blocks, n_vis, wa, idx_loc,
                    idx_anc, idx_dyn);
}

cudaError_t launch_fuse3(float* o, const float* o_loc, const float* o_anc, const float* gates, int T, int sm_count,
                         cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const long long n4 = (long long)T * 64 * 512 / 4;
  const long long want = (n4 + 255) / 256;
  const int grid = int(want < 8LL * sm_count ? want : 8LL * sm_count);
  return launch_pdl(fuse3_kernel, dim3(unsigned(grid)), dim3(256), 0, stream, 1, o, o_loc, o_anc, gates, n4);
}

}  // namespace dsa
