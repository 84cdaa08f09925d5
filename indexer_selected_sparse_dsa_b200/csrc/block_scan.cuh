// Warp- and block-wide scans used by the planning and selection kernels.
#pragma once
#include <cstdint>

namespace dsa {

template <class T>
__device__ __forceinline__ T warp_inclusive_sum(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

template <class T>
__device__ __forceinline__ T warp_inclusive_max(T v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    T n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v = n > v ? n : v;
  }
  return v;
}

// Block-wide exclusive prefix sum over blockDim.x threads (a multiple of 32, <= 1024).
// `scratch` holds >= 33 elements of shared memory.  Returns the exclusive prefix and
// writes the block total to *total.  Contains __syncthreads(); every thread must call.
template <class T>
__device__ __forceinline__ T block_exclusive_sum(T v, T* scratch, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  T inc = warp_inclusive_sum(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    T s = lane < nw ? scratch[lane] : T(0);
    T si = warp_inclusive_sum(s);
    if (lane < nw) scratch[lane] = si - s;
    if (lane == nw - 1) scratch[32] = si;
  }
  __syncthreads();
  T out = scratch[warp] + inc - v;
  *total = scratch[32];
  __syncthreads();
  return out;
}

// Block-wide inclusive prefix max (same contract as above).
template <class T>
__device__ __forceinline__ T block_inclusive_max(T v, T* scratch, T identity) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  T inc = warp_inclusive_max(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    T s = lane < nw ? scratch[lane] : identity;
    T si = warp_inclusive_max(s);
    // exclusive max for each warp
    T ex = __shfl_up_sync(0xffffffffu, si, 1);
    if (lane == 0) ex = identity;
    if (lane < nw) scratch[lane] = ex;
  }
  __syncthreads();
  T pre = scratch[warp];
  T out = pre > inc ? pre : inc;
  __syncthreads();
  return out;
}

}  // namespace dsa
