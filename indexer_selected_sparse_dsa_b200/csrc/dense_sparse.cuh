// Dense + sparse attention: the two branches of a DSA layer and their fusion.
//
// ("GLM-5.2's DSA architecture: how dense and sparse attention split the work",
// section "DSA's core design: dense and sparse side by side": each layer runs
// local dense attention over a sliding window next to the current token and
// global sparse attention over the selected top-k positions, and fuses the two
// outputs with learned weights.)  The sparse branch is the sparse MLA kernel
// over the selected positions; the dense branch is the same kernel over the
// window positions n - window .. n - 1, listed by window_idx_kernel; the
// fusion takes a per-(row, head) gate from the caller:
//     o = gate * o_dense + (1 - gate) * o_sparse.
#pragma once
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

// idx_w[i, j] = n_vis[i] - window + j, or -1 where that is negative (rows shorter
// than the window); ascending, like every index row of the library.
__global__ void window_idx_kernel(const int32_t* __restrict__ n_vis, int T, int window, int32_t* __restrict__ idx_w) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x;
  const int n = n_vis[i];
  if (n < 1 && threadIdx.x == 0) raise_status(kStatusBadRow);
  int32_t* row = idx_w + (long long)i * window;
  for (int j = threadIdx.x; j < window; j += blockDim.x) {
    const int p = n - window + j;
    row[j] = (n >= 1 && p >= 0) ? p : -1;
  }
}

// o[i,h,:] = gate[i,h] * o_dense[i,h,:] + (1 - gate[i,h]) * o[i,h,:], in place.
__global__ void fuse_kernel(float* __restrict__ o, const float* __restrict__ o_dense, const float* __restrict__ gate,
                            long long n4) {
  pdl_wait();
  pdl_trigger();
  for (long long v = blockIdx.x * (long long)blockDim.x + threadIdx.x; v < n4; v += (long long)gridDim.x * blockDim.x) {
    const float g = gate[(v * 4) >> 9];  // 512 latent dims per (row, head)
    const float4 d = reinterpret_cast<const float4*>(o_dense)[v];
    float4 s = reinterpret_cast<float4*>(o)[v];
    s.x = fmaf(g, d.x - s.x, s.x);
    s.y = fmaf(g, d.y - s.y, s.y);
    s.z = fmaf(g, d.z - s.z, s.z);
    s.w = fmaf(g, d.w - s.w, s.w);
    reinterpret_cast<float4*>(o)[v] = s;
  }
}

}  // namespace

cudaError_t launch_window_idx(const int32_t* n_vis, int T, int window, int32_t* idx_w, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  return launch_pdl(window_idx_kernel, dim3(unsigned(T)), dim3(256), 0, stream, 1, n_vis, T, window, idx_w);
}

cudaError_t launch_fuse(float* o, const float* o_dense, const float* gate, int T, int sm_count, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const long long n4 = (long long)T * 64 * 512 / 4;
  const long long want = (n4 + 255) / 256;
  const int grid = int(want < 8LL * sm_count ? want : 8LL * sm_count);
  return launch_pdl(fuse_kernel, dim3(unsigned(grid)), dim3(256), 0, stream, 1, o, o_dense, gate, n4);
}

}  // namespace dsa
