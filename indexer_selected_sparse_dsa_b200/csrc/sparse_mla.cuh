// Sparse MLA attention in latent (absorbed) form over the selected rows.
//
//   S[h,j]   = scale * (q_lat[h] . c_kv[s_j] + q_rope[h] . k_rope[s_j])
//   o_lat[h] = sum_j softmax_j(S[h,:]) c_kv[s_j],   lse[h] = log sum_j exp S[h,j]
//
// ("From a trillion dot products to two thousand: how DSA breaks N^2", "DSA full flow": full Q.K, softmax and the
// value mix over the selected 2048 only; "2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.1: 64 heads, kv_lora_rank 512, rope 64, qk_head_dim 256.)
//
// One CTA per query row.  The selected 1152-byte rows are gathered 128 at a
// time with 16-byte cp.async into a 128-byte-swizzled tile (9 column chunks
// of 64).  Each tile is used twice by the tensor cores without moving it:
//  * S^T = K . Q^T   (M = 128 keys, N = 64 heads, K = 576): A = tile, K-major;
//    B = q (resident, 9 chunks), K-major.  S^T lands in TMEM: lane = key.
//  * O^T += V^T . P^T (M = 128 latent dims x 4, N = 64 heads, K = 128 keys):
//    A = the same tile read MN-major (the latent dims are contiguous), B = P
//    written as bf16 into the tile's rope chunk, which is dead once S exists.
// Softmax state is fp32: each thread owns one key row of S^T; the per-head
// max and sum across the 128 keys use a 62-shuffle reduce-scatter per warp
// plus a 4-way combine in shared memory.  The running max is updated lazily
// (only when a tile max exceeds it by 2^8), so O in TMEM is rescaled rarely.
#pragma once
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kRow = 576;
constexpr int kTileKeys = 128;
constexpr int kChunkKeyBytes = kTileKeys * 128;  // 16 KB: 128 rows x 64 columns
constexpr int kQChunkBytes = 64 * 128;           // 8 KB: 64 heads x 64 columns
constexpr int kTileOff = 0;
constexpr int kQOff = 9 * kChunkKeyBytes;                // 147456
constexpr int kMiscOff = kQOff + 9 * kQChunkBytes;       // 221184
constexpr int kRedOff = kMiscOff;                        // float red[4][64]
constexpr int kMUseOff = kRedOff + 4 * 64 * 4;           // float m_use[64]
constexpr int kLOff = kMUseOff + 64 * 4;                 // float l_run[64]
constexpr int kAlphaOff = kLOff + 64 * 4;                // float alpha[64]
constexpr int kIdxOff = kAlphaOff + 64 * 4;              // long long row[128] (absolute cache row or -1)
constexpr int kBarOff = kIdxOff + 128 * 8;               // 5 mbarriers
constexpr int kSlotOff = kBarOff + 5 * 8;                // tmem slot, abort flag
constexpr int kSmemBytes = kSlotOff + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;    // S^T: 64 columns
constexpr uint32_t kOCol = 64;   // O^T: 4 tiles x 64 columns
constexpr float kLazyRescale = 8.0f;  // log2 units

__device__ __forceinline__ float fmax_(float a, float b) { return a > b ? a : b; }

// Reduce 64 per-thread values across the warp; lane L returns heads 2L, 2L+1.
template <bool kMax>
__device__ __forceinline__ void reduce_scatter64(const float (&v)[64], float& r0, float& r1) {
  const int lane = threadIdx.x & 31;
  float a[32];
  {
    const bool up = lane & 16;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float mine = up ? v[32 + i] : v[i];
      const float give = up ? v[i] : v[32 + i];
      const float got = __shfl_xor_sync(0xffffffffu, give, 16);
      a[i] = kMax ? fmax_(mine, got) : mine + got;
    }
  }
  float b[16];
  {
    const bool up = lane & 8;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const float mine = up ? a[16 + i] : a[i];
      const float give = up ? a[i] : a[16 + i];
      const float got = __shfl_xor_sync(0xffffffffu, give, 8);
      b[i] = kMax ? fmax_(mine, got) : mine + got;
    }
  }
  float c[8];
  {
    const bool up = lane & 4;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float mine = up ? b[8 + i] : b[i];
      const float give = up ? b[i] : b[8 + i];
      const float got = __shfl_xor_sync(0xffffffffu, give, 4);
      c[i] = kMax ? fmax_(mine, got) : mine + got;
    }
  }
  float d[4];
  {
    const bool up = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float mine = up ? c[4 + i] : c[i];
      const float give = up ? c[i] : c[4 + i];
      const float got = __shfl_xor_sync(0xffffffffu, give, 2);
      d[i] = kMax ? fmax_(mine, got) : mine + got;
    }
  }
  {
    const bool up = lane & 1;
    float e[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float mine = up ? d[2 + i] : d[i];
      const float give = up ? d[i] : d[2 + i];
      const float got = __shfl_xor_sync(0xffffffffu, give, 1);
      e[i] = kMax ? fmax_(mine, got) : mine + got;
    }
    r0 = e[0];
    r1 = e[1];
  }
}

__device__ __forceinline__ int bar_red_or_128(int pred) {
  int out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.s32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, 1, 128, pi;\n\t"
      "selp.s32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(pred)
      : "memory");
  return out;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi, float& rlo, float& rhi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  rlo = __low2float(p);
  rhi = __high2float(p);
  return *reinterpret_cast<uint32_t*>(&p);
}

__global__ void __launch_bounds__(160, 1)
    sparse_mla_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ kv, int64_t cache_rows,
                      const int64_t* __restrict__ kv_start, const int32_t* __restrict__ idx, int topk,
                      float scale_log2, float* __restrict__ o_lat, float* __restrict__ lse, WaitLimit lim) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  float* red = reinterpret_cast<float*>(smem + kRedOff);
  float* m_use = reinterpret_cast<float*>(smem + kMUseOff);
  float* l_run = reinterpret_cast<float*>(smem + kLOff);
  float* alpha_s = reinterpret_cast<float*>(smem + kAlphaOff);
  long long* row_s = reinterpret_cast<long long*>(smem + kIdxOff);
  const uint32_t kv_full = sbase + kBarOff, s_full = kv_full + 8, p_full = kv_full + 16, kv_free = kv_full + 24;
  const uint32_t drain = kv_full + 32;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSlotOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int ntiles = (topk + kTileKeys - 1) / kTileKeys;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 128);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(kv_free, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < 64) {
    m_use[threadIdx.x] = -INFINITY;
    l_run[threadIdx.x] = 0.f;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_o = idesc_bf16(128, 64, 1, 1);
      const uint32_t tile = sbase + kTileOff, qs = sbase + kQOff, pbuf = tile + 8 * kChunkKeyBytes;
      for (int t = 0; t < ntiles; ++t) {
        if (!mbar_wait(kv_full, uint32_t(t & 1), lim, abort_flag)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 9; ++c)
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = smem_desc(tile + c * kChunkKeyBytes + k * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(qs + c * kQChunkBytes + k * 32, 16, 1024, kSwizzle128B);
            mma_bf16_ss(tmem + kSCol, ad, bd, idesc_s, (c | k) ? 1u : 0u);
          }
        mma_commit(s_full);
        if (!mbar_wait(p_full, uint32_t(t & 1), lim, abort_flag)) break;
        tc_fence_after();
#pragma unroll 1
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // V^T tile m: latent dims 128m..128m+127 are chunks 2m, 2m+1 (LBO apart); keys 16k..16k+15.
            const uint64_t ad = smem_desc(tile + (2 * m) * kChunkKeyBytes + k * 2048, kChunkKeyBytes, 1024,
                                          kSwizzle128B);
            const uint64_t bd = smem_desc(pbuf + k * 2048, kChunkKeyBytes, 1024, kSwizzle128B);
            mma_bf16_ss(tmem + kOCol + 64 * m, ad, bd, idesc_o, (t > 0 || k > 0) ? 1u : 0u);
          }
        mma_commit(kv_free);
      }
      // every MMA issued above must be complete before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, lim, nullptr);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- gather + softmax (warps 0..3)
    const int st = threadIdx.x;  // 0..127
    const int quarter = warp;    // TMEM lane quarter
    const int r = quarter * 32 + lane;
    const long long ks = kv_start[i];
    const int32_t* irow = idx + (long long)i * topk;
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      if (t > 0 && !mbar_wait(kv_free, uint32_t((t - 1) & 1), lim, abort_flag)) {
        ok = false;
        break;
      }
      // stage this tile's cache rows
      {
        const int slot = t * kTileKeys + st;
        long long rr = -1;
        if (slot < topk) {
          const int s = irow[slot];
          if (s >= 0) {
            if (ks + s < cache_rows) rr = ks + s;
            else raise_status(kStatusBadRow);
          }
        }
        row_s[st] = rr;
      }
      named_bar_sync(1, 128);
      if (t == 0) {
        const uint16_t* qrow = q + (long long)i * 64 * kRow;
        for (int e = st; e < 64 * 72; e += 128) {
          const int h = e / 72, rem = e - h * 72, c = rem >> 3, g = rem & 7;
          const uint32_t dst = sbase + kQOff + c * kQChunkBytes + h * 128 + ((g ^ (h & 7)) << 4);
          cp_async_16(dst, qrow + h * kRow + c * 64 + g * 8, true);
        }
      }
      for (int e = st; e < kTileKeys * 72; e += 128) {
        const int row = e / 72, rem = e - row * 72, c = rem >> 3, g = rem & 7;
        const long long rr = row_s[row];
        const uint32_t dst = sbase + kTileOff + c * kChunkKeyBytes + row * 128 + ((g ^ (row & 7)) << 4);
        const uint16_t* src = rr >= 0 ? kv + rr * kRow + c * 64 + g * 8 : kv;
        cp_async_16(dst, src, rr >= 0);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(kv_full);

      if (!mbar_wait(s_full, uint32_t(t & 1), lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float x[64];
      const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
      tmem_ld32_sync(lane_addr + kSCol, x);
      tmem_ld32_sync(lane_addr + kSCol + 32, x + 32);
      const bool valid = row_s[r] >= 0;
#pragma unroll
      for (int h = 0; h < 64; ++h) x[h] = valid ? x[h] * scale_log2 : -INFINITY;

      // per-head max over the tile's 128 keys
      float r0, r1;
      reduce_scatter64<true>(x, r0, r1);
      red[quarter * 64 + 2 * lane] = r0;
      red[quarter * 64 + 2 * lane + 1] = r1;
      named_bar_sync(1, 128);
      int resc = 0;
      if (st < 64) {
        const float mt = fmax_(fmax_(red[st], red[64 + st]), fmax_(red[128 + st], red[192 + st]));
        const float mu = m_use[st];
        float al = 1.f;
        if (mt > -INFINITY && (mu == -INFINITY || mt > mu + kLazyRescale)) {
          al = exp2f(mu - mt);  // 0 when mu = -inf
          m_use[st] = mt;
          l_run[st] *= al;
          resc = (t > 0) && (al != 1.f);
        }
        alpha_s[st] = al;
      }
      resc = bar_red_or_128(resc);  // also the barrier that publishes m_use / alpha

      // probabilities (bf16 for the MMA) and their per-head sums
      float p[64];
      uint8_t* prow = smem + kTileOff + 8 * kChunkKeyBytes + r * 128;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        uint32_t w4[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h = g * 8 + 2 * u;
          const float m0 = m_use[h], m1 = m_use[h + 1];
          const float e0 = (valid && m0 > -INFINITY) ? exp2f(x[h] - m0) : 0.f;
          const float e1 = (valid && m1 > -INFINITY) ? exp2f(x[h + 1] - m1) : 0.f;
          w4[u] = pack_bf16x2(e0, e1, p[h], p[h + 1]);
        }
        *reinterpret_cast<uint4*>(prow + ((g ^ (r & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
      }
      reduce_scatter64<false>(p, r0, r1);
      red[quarter * 64 + 2 * lane] = r0;
      red[quarter * 64 + 2 * lane + 1] = r1;

      if (resc) {
        // O^T (lane = latent dim, column = head) *= alpha[head]; PV(t-1) is complete.
#pragma unroll 1
        for (int m = 0; m < 4; ++m)
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            float o[32];
            const uint32_t a = lane_addr + kOCol + 64 * m + 32 * half;
            tmem_ld32_sync(a, o);
#pragma unroll
            for (int h = 0; h < 32; ++h) o[h] *= alpha_s[32 * half + h];
            tmem_st16(a, o);
            tmem_st16(a + 16, o + 16);
          }
        tmem_wait_st();
      }
      named_bar_sync(1, 128);
      if (st < 64) l_run[st] += red[st] + red[64 + st] + red[128 + st] + red[192 + st];
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // final PV must be complete before reading O
    if (ok && ntiles > 0) ok = mbar_wait(kv_free, uint32_t((ntiles - 1) & 1), lim, abort_flag);
  }
  // All 160 threads (the MMA warp after its drain): publishes l_run / m_use and
  // makes the abort decision uniform before the epilogue.
  __syncthreads();
  if (warp < 4 && !*abort_flag) {
    const int st = threadIdx.x;
    const int quarter = warp;
    {
      tc_fence_after();
      const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
      float* orow = o_lat + (long long)i * 64 * 512;
#pragma unroll 1
      for (int m = 0; m < 4; ++m) {
        const int d = 128 * m + quarter * 32 + lane;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          float o[32];
          tmem_ld32_sync(lane_addr + kOCol + 64 * m + 32 * half, o);
#pragma unroll
          for (int hh = 0; hh < 32; ++hh) {
            const int h = 32 * half + hh;
            const float l = l_run[h];
            orow[h * 512 + d] = l > 0.f ? o[hh] / l : 0.f;
          }
        }
      }
      if (lse && st < 64) {
        const float l = l_run[st];
        lse[(long long)i * 64 + st] = l > 0.f ? (m_use[st] + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t prepare_sparse_mla() {
  static_assert(kSmemAlloc <= 232448, "sparse MLA shared memory exceeds the per-CTA limit");
  return cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
}

cudaError_t launch_sparse_mla(const MlaLaunch& p) {
  if (p.T <= 0) return cudaSuccess;
  const float scale_log2 = p.scale * 1.4426950408889634f;
  sparse_mla_kernel<<<p.T, 160, kSmemAlloc, p.stream>>>(p.q, p.kv, p.cache_rows, p.kv_start, p.idx, p.topk,
                                                        scale_log2, p.o_lat, p.lse, WaitLimit{p.wait_ns});
  return cudaGetLastError();
}

}  // namespace dsa
