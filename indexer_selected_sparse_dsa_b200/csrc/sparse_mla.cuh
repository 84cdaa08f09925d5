// Sparse MLA attention in latent (absorbed) form over the selected rows.
//
//   S[h,j]   = scale * (q_lat[h] . c_kv[s_j] + q_rope[h] . k_rope[s_j])
//   o_lat[h] = sum_j softmax_j(S[h,:]) c_kv[s_j],   lse[h] = log sum_j exp S[h,j]
//
// ("From a trillion dot products to two thousand: how DSA breaks N^2", "DSA
// full flow": full Q.K, softmax and the value mix over the selected 2048
// only; "2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2",
// section 2.1: 64 heads, kv_lora_rank 512, rope 64, qk_head_dim 256.)
//
// One CTA per (query row, split of its selected positions); 9 warps:
//  * warps 0..3, producers: q (64 x 576) once by TMA, then a stream of 32 KB
//    slots through a 4-deep ring.  A slot is two 64-column chunks of 128
//    selected rows in the 128-byte-swizzled layout the tensor cores read,
//    filled with 16-byte cp.async (an empty index slot is zero-filled); each
//    thread's copies arrive on the slot's mbarrier when they land, so every
//    free slot of the ring is in flight; the selected positions are read two
//    tiles ahead.  (An L2 prefetch of the next tile's rows measured slower:
//    the bulk prefetches queue ahead of the copies.)  Per tile t the stream
//    carries its key chunks 0..8 (five slots) and, one tile later, its latent
//    chunks 0..7 again (four slots) for the value product: the rows cross L2
//    twice instead of holding a 144 KB tile.
//  * warp 4, MMA issuer: S^T_t = K_t . Q^T (M = 128 keys, N = 64 heads,
//    K = 576) into one of two TMEM buffers, one tile ahead of
//    O^T += V_t^T . P_t^T (M = 128 latent dims x 4, N = 64, K = 128), with V
//    read MN-major straight from the slot.
//  * warps 5..8, softmax: each thread owns one key row of S^T.  Exponents are
//    taken against a lazily updated running max: each thread checks its own
//    row against it, and only when some score passes it by 2^8 (one barrier
//    vote) is the tile max reduced across the CTA and O rescaled.  Each thread
//    keeps its row's share of the running sums in registers; they are reduced
//    once after the last tile.  P goes to shared memory as bf16 for the value
//    product.
#pragma once
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kRow = 576;
constexpr int kTileKeys = 128;
constexpr int kChunkBytes = kTileKeys * 128;     // 16 KB: 128 rows x 64 columns, 128B-swizzled
constexpr int kSlotBytes = 2 * kChunkBytes;      // two chunks
constexpr int kNumSlots = 4;
constexpr int kQChunkBytes = 64 * 128;           // 8 KB: 64 heads x 64 columns
constexpr int kKeySlots = 5;                     // chunks 0..8 of a key tile
constexpr int kValSlots = 4;                     // chunks 0..7 of a value tile
constexpr int kQOff = 0;                                    // 9 x 8 KB
constexpr int kRingOff = 9 * kQChunkBytes;                  // 73728
constexpr int kPOff = kRingOff + kNumSlots * kSlotBytes;    // 204800: P, 128 keys x 64 heads bf16
constexpr int kMiscOff = kPOff + kChunkBytes;               // 221184
constexpr int kRedOff = kMiscOff;                           // float red[4][64]
constexpr int kMUseOff = kRedOff + 4 * 64 * 4;              // float m_use[64]
constexpr int kLOff = kMUseOff + 64 * 4;                    // float l_run[64]
constexpr int kAlphaOff = kLOff + 64 * 4;                   // float alpha[64]
constexpr int kYOff = kAlphaOff + 64 * 4;                   // int y[2][128]: cache rows of two tiles
constexpr int kBarOff = kYOff + 2 * 128 * 4;                // mbarriers
constexpr int kNumBars = 1 + 2 * kNumSlots + 2 + 1 + 1 + 1; // q, slots full/empty, s_full x2, p_full, p_free, drain
constexpr int kSlotOff = kBarOff + kNumBars * 8;            // tmem slot, abort flag
constexpr int kSmemBytes = kSlotOff + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 0;     // S^T buffers: columns 0..63 and 64..127
constexpr uint32_t kOCol = 128;   // O^T: 4 tiles x 64 columns
constexpr float kLazyRescale = 8.0f;  // log2 units
constexpr int kPartFloats = 64 * 512 + 2 * 64;  // one split's O, running max, running sum
constexpr int kMlaThreads = 288;

__device__ __forceinline__ float fmax_(float a, float b) { return a > b ? a : b; }

// 2^x with the SFU instruction (ex2.approx: relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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

// bar.red.or over `nthreads` threads on named barrier `id`: 1 when any of them has pred != 0.
__device__ __forceinline__ int bar_red_or(int id, int nthreads, int pred) {
  int out;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.s32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.s32 %0, 1, 0, po;\n\t}"
      : "=r"(out)
      : "r"(pred), "r"(id), "r"(nthreads)
      : "memory");
  return out;
}
__device__ __forceinline__ int bar_red_or_128(int pred) { return bar_red_or(1, 128, pred); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi, float& rlo, float& rhi) {
  __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  rlo = __low2float(p);
  rhi = __high2float(p);
  return *reinterpret_cast<uint32_t*>(&p);
}

__global__ void __launch_bounds__(kMlaThreads, 1)
    sparse_mla_kernel(const uint16_t* __restrict__ kv, const __grid_constant__ CUtensorMap tmap_q,
                      int64_t cache_rows, const int64_t* __restrict__ kv_start, const int32_t* __restrict__ idx,
                      int topk, float scale_log2, float* __restrict__ o_lat, float* __restrict__ lse, int splits,
                      int tiles_per_split, float* __restrict__ part, WaitLimit lim) {
  extern __shared__ uint8_t smem_raw[];
  // 1 KB-aligned base by pointer arithmetic on the shared array (an integer round trip
  // would hide the shared address space and turn every access into a generic one)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float* red = reinterpret_cast<float*>(smem + kRedOff);
  float* m_use = reinterpret_cast<float*>(smem + kMUseOff);
  float* l_run = reinterpret_cast<float*>(smem + kLOff);
  float* alpha_s = reinterpret_cast<float*>(smem + kAlphaOff);
  const uint32_t bar0 = sbase + kBarOff;
  const uint32_t q_full = bar0;
  auto slot_full = [&](int j) { return bar0 + 8u * (1 + j); };
  auto slot_empty = [&](int j) { return bar0 + 8u * (1 + kNumSlots + j); };
  auto s_full = [&](int b) { return bar0 + 8u * (1 + 2 * kNumSlots + b); };
  const uint32_t p_full = bar0 + 8u * (3 + 2 * kNumSlots);
  const uint32_t p_free = bar0 + 8u * (4 + 2 * kNumSlots);
  const uint32_t drain = bar0 + 8u * (5 + 2 * kNumSlots);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kSlotOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // CTA = (query row i, split sp); the split owns tiles [t_first, t_first + ntiles).
  const int i = blockIdx.x / splits;
  const int sp = blockIdx.x - i * splits;
  const int ntiles_row = (topk + kTileKeys - 1) / kTileKeys;
  const int t_first = sp * tiles_per_split;
  const int ntiles = max(0, min(ntiles_row, t_first + tiles_per_split) - t_first);
  const int32_t* irow = idx + (long long)i * topk;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int j = 0; j < kNumSlots; ++j) {
      mbar_init(slot_full(j), 128);  // one arrival per producer thread
      mbar_init(slot_empty(j), 1);
    }
    mbar_init(s_full(0), 1);
    mbar_init(s_full(1), 1);
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_q);
  }
  if (threadIdx.x >= 160 && threadIdx.x < 224) {
    m_use[threadIdx.x - 160] = -INFINITY;
    l_run[threadIdx.x - 160] = 0.f;
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // everything above touched shared memory and TMEM only
  const long long ks = kv_start[i];

  if (warp < 4) {
    // ---------------------------------------------------------------- producers (warps 0..3)
    const int pt = threadIdx.x;  // 0..127
    int* y_s = reinterpret_cast<int*>(smem + kYOff);
    if (pt == 0 && ntiles > 0) {
      mbar_arrive_expect_tx(q_full, 9 * kQChunkBytes);
      for (int c = 0; c < 9; ++c) tma_load_2d(sbase + kQOff + c * kQChunkBytes, &tmap_q, q_full, 64 * c, i * 64);
    }
    // Thread pt copies 16-byte segment g of chunk half h for rows r + 8j (j < 16), in
    // every slot: the swizzled destination offset is the same for all its rows.
    const int h = (pt >> 3) & 1, g = pt & 7, r = pt >> 4;
    const uint32_t thr_off = uint32_t(h * kChunkBytes + r * 128 + ((g ^ (r & 7)) << 4));
    const char* kvb = reinterpret_cast<const char*>(kv);
    const char* cur[16];
    const char* prev[16];
    uint32_t cur_skip = 0u, prev_skip = 0u;  // bit j: row r + 8j is empty (zero-filled)
    int slot = 0;
    uint32_t sphase = 0;
    bool ok = true;
    // copy chunk `chunk` (plus h) of the rows in `rows` into the next slot
    auto issue_slot = [&](int chunk, bool active, const char* const* rows, uint32_t skip) {
      if (!mbar_wait(slot_empty(slot), sphase ^ 1u, lim, abort_flag)) return false;
      if (active) {
        const uint32_t dst = sbase + kRingOff + slot * kSlotBytes + thr_off;
        const int col = (chunk + h) * 128 + g * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) cp_async_16_or_zero(dst + j * 1024, rows[j] + col, (skip >> j) & 1u);
      }
      cp_async_arrive_noinc(slot_full(slot));  // arrives when this thread's copies have landed
      if (++slot == kNumSlots) {
        slot = 0;
        sphase ^= 1u;
      }
      return true;
    };
    // Selected positions run two tiles ahead in registers (one key row per
    // thread), so staging a tile never waits on a global load.
    auto load_pos = [&](int tile) {
      const int slot_i = (t_first + tile) * kTileKeys + pt;
      return (tile < ntiles && slot_i < topk) ? irow[slot_i] : -1;
    };
    int v0 = load_pos(0), v1 = load_pos(1);
    for (int s = 0; s <= ntiles; ++s) {
      // Every producer is done reading y_s for the previous tile, and all of them
      // agree whether to go on: a wait that failed in any one ends the loop for all
      // (none is left behind at the named barrier below).
      if (bar_red_or(2, 128, ok ? 0 : 1)) {
        ok = false;
        break;
      }
      if (s < ntiles) {
        // cache rows of tile s (-1: empty or out of range) into y_s[s & 1]
        {
          int yy = -1;
          if (v0 >= 0) {
            if (ks + v0 < cache_rows) yy = int(ks + v0);
            else raise_status(kStatusBadRow);
          }
          y_s[(s & 1) * 128 + pt] = yy;
          v0 = v1;
          v1 = load_pos(s + 2);
        }
        named_bar_sync(2, 128);
        cur_skip = 0u;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int y = y_s[(s & 1) * 128 + r + 8 * j];
          cur[j] = kvb + (long long)(y >= 0 ? y : 0) * (kRow * 2);
          cur_skip |= (y < 0 ? 1u : 0u) << j;
        }
#pragma unroll
        for (int p = 0; p < kKeySlots; ++p)
          if (ok) ok = issue_slot(2 * p, p < 4 || h == 0, cur, cur_skip);  // the rope slot has one chunk
      }
      if (s >= 1) {
#pragma unroll
        for (int p = 0; p < kValSlots; ++p)
          if (ok) ok = issue_slot(2 * p, true, prev, prev_skip);
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) prev[j] = cur[j];
      prev_skip = cur_skip;
    }
    cp_async_wait_all();  // no copy may still be in flight when the CTA exits
    if (pt == 0 && ntiles > 0) mbar_drain(q_full, 0);  // nor the query tile (an abort may leave it unread)
  } else if (warp == 4) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && ntiles > 0) {
      const uint32_t idesc_s = idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_o = idesc_bf16(128, 64, 1, 1);
      int slot = 0;
      uint32_t sphase = 0;
      bool ok = mbar_wait(q_full, 0, lim, abort_flag);
      for (int s = 0; s <= ntiles && ok; ++s) {
        if (s < ntiles) {
          const uint32_t d = tmem + kSCol + 64 * (s & 1);
          for (int p = 0; p < kKeySlots && ok; ++p) {
            if (!(ok = mbar_wait(slot_full(slot), sphase, lim, abort_flag))) break;
            tc_fence_after();
            const uint32_t a0 = sbase + kRingOff + slot * kSlotBytes;
            const int nch = p < 4 ? 2 : 1;
            for (int h = 0; h < nch; ++h) {
              const int c = 2 * p + h;
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t ad = smem_desc(a0 + h * kChunkBytes + 32 * k, 16, 1024, kSwizzle128B);
                const uint64_t bd = smem_desc(sbase + kQOff + c * kQChunkBytes + 32 * k, 16, 1024, kSwizzle128B);
                mma_bf16_ss(d, ad, bd, idesc_s, (c | k) ? 1u : 0u);
              }
            }
            mma_commit(slot_empty(slot));
            if (++slot == kNumSlots) {
              slot = 0;
              sphase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(s_full(s & 1));
        }
        if (s >= 1) {
          const int t = s - 1;
          if (!(ok = mbar_wait(p_full, uint32_t(t & 1), lim, abort_flag))) break;
          tc_fence_after();
          for (int m = 0; m < kValSlots && ok; ++m) {
            if (!(ok = mbar_wait(slot_full(slot), sphase, lim, abort_flag))) break;
            tc_fence_after();
            const uint32_t a0 = sbase + kRingOff + slot * kSlotBytes;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              // V^T: latent dims 128m..128m+127 = the slot's two chunks (LBO apart); keys 16k..16k+15
              const uint64_t ad = smem_desc(a0 + k * 2048, kChunkBytes, 1024, kSwizzle128B);
              const uint64_t bd = smem_desc(sbase + kPOff + k * 2048, kChunkBytes, 1024, kSwizzle128B);
              mma_bf16_ss(tmem + kOCol + 64 * m, ad, bd, idesc_o, (t > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(slot_empty(slot));
            if (++slot == kNumSlots) {
              slot = 0;
              sphase ^= 1u;
            }
          }
          if (!ok) break;
          mma_commit(p_free);
        }
      }
      // every MMA issued above must be complete before TMEM is released
      mma_commit(drain);
      mbar_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax (warps 5..8)
    const int st = threadIdx.x - 160;  // 0..127
    const int quarter = warp & 3;     // TMEM lane quarter
    const int r = quarter * 32 + lane;
    const int rw = st >> 5;           // slot of this warp in red[]
    const uint32_t lane_addr = tmem + (uint32_t(quarter * 32) << 16);
    // This thread's share of each head's running sum (its key row over all
    // tiles); reduced across the 128 threads once, after the last tile.
    float l_acc[64];
#pragma unroll
    for (int h = 0; h < 64; ++h) l_acc[h] = 0.f;
    // One softmax thread waits on the mbarrier; the barrier reduction then hands
    // every softmax thread both the outcome and the memory ordering, so a failed
    // wait ends the loop for all of them at the same point, before any named
    // barrier inside it.
    auto wait_all = [&](uint32_t bar, uint32_t parity) {
      const bool mine = st == 0 ? mbar_wait(bar, parity, lim, abort_flag) : true;
      return bar_red_or_128(mine ? 0 : 1) == 0;
    };
    bool ok = true;
    for (int t = 0; t < ntiles && ok; ++t) {
      const int slot_i = (t_first + t) * kTileKeys + r;
      bool valid = false;
      if (slot_i < topk) {
        const int s = irow[slot_i];
        valid = s >= 0 && ks + s < cache_rows;
      }
      if (!(ok = wait_all(s_full(t & 1), uint32_t((t >> 1) & 1)))) break;
      tc_fence_after();
      // Lazy running max: exponents stay taken against m_use while no score of
      // the tile passes it by more than 2^kLazyRescale, which each thread checks
      // for its own key row; only then is the tile max reduced and O rescaled.
      int above = 0;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float y[32];
        tmem_ld32_sync(lane_addr + kSCol + 64 * (t & 1) + 32 * half, y);
#pragma unroll
        for (int h = 0; h < 32; ++h) above |= (valid && y[h] * scale_log2 > m_use[32 * half + h] + kLazyRescale) ? 1 : 0;
      }
      int resc = 0;
      if (bar_red_or_128(above)) {
        float x[64];
        tmem_ld32_sync(lane_addr + kSCol + 64 * (t & 1), x);
        tmem_ld32_sync(lane_addr + kSCol + 64 * (t & 1) + 32, x + 32);
#pragma unroll
        for (int h = 0; h < 64; ++h) x[h] = valid ? x[h] * scale_log2 : -INFINITY;
        float r0, r1;
        reduce_scatter64<true>(x, r0, r1);
        red[rw * 64 + 2 * lane] = r0;
        red[rw * 64 + 2 * lane + 1] = r1;
        named_bar_sync(1, 128);
        int mine = 0;
        if (st < 64) {
          const float mt = fmax_(fmax_(red[st], red[64 + st]), fmax_(red[128 + st], red[192 + st]));
          const float mu = m_use[st];
          float al = 1.f;
          if (mt > -INFINITY && (mu == -INFINITY || mt > mu + kLazyRescale)) {
            al = fast_exp2(mu - mt);  // 0 when mu = -inf
            m_use[st] = mt;
            mine = (t > 0) && (al != 1.f);
          }
          alpha_s[st] = al;
        }
        resc = bar_red_or_128(mine);  // also the barrier that publishes m_use / alpha
      }

      // the single P buffer and O are free once the previous value product is done
      if (t > 0 && !(ok = wait_all(p_free, uint32_t((t - 1) & 1)))) break;
      if (resc) {
        tc_fence_after();
        // O^T (lane = latent dim, column = head) *= alpha[head]
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
#pragma unroll
        for (int h = 0; h < 64; ++h) l_acc[h] *= alpha_s[h];
      }
      // probabilities (bf16 for the MMA); the sums take the same rounded values.
      // S is read from TMEM again, 32 heads at a time: this tile's buffer is
      // not overwritten before P is published (the next QK into it is issued
      // after this tile's value product).
      uint8_t* prow = smem + kPOff + r * 128;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float y[32];
        tmem_ld32_sync(lane_addr + kSCol + 64 * (t & 1) + 32 * half, y);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t w4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int hl = g * 8 + 2 * u, h = 32 * half + hl;
            const float m0 = m_use[h], m1 = m_use[h + 1];
            const float e0 = (valid && m0 > -INFINITY) ? fast_exp2(y[hl] * scale_log2 - m0) : 0.f;
            const float e1 = (valid && m1 > -INFINITY) ? fast_exp2(y[hl + 1] * scale_log2 - m1) : 0.f;
            float q0, q1;
            w4[u] = pack_bf16x2(e0, e1, q0, q1);
            l_acc[h] += q0;
            l_acc[h + 1] += q1;
          }
          const int gg = 4 * half + g;
          *reinterpret_cast<uint4*>(prow + ((gg ^ (r & 7)) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // the last value product must be complete before O is read
    if (ok && ntiles > 0) ok = wait_all(p_free, uint32_t((ntiles - 1) & 1));
    if (ok) {  // the same in all softmax threads
      // running sums: one reduction over the tile rows
      float r0, r1;
      reduce_scatter64<false>(l_acc, r0, r1);
      red[rw * 64 + 2 * lane] = r0;
      red[rw * 64 + 2 * lane + 1] = r1;
      named_bar_sync(1, 128);
      if (st < 64) l_run[st] = red[st] + red[64 + st] + red[128 + st] + red[192 + st];
      named_bar_sync(1, 128);  // publishes l_run (and the last m_use) to the four warps
      tc_fence_after();
      // one split: the normalised output; several: this split's unnormalised O with
      // its running max (log2 units) and sum, merged by sparse_mla_combine_kernel
      const bool direct = (splits == 1);
      float* orow = direct ? o_lat + (long long)i * 64 * 512 : part + (long long)blockIdx.x * kPartFloats;
      if (ntiles == 0) {
        for (int e = st; e < 64 * 512; e += 128) orow[e] = 0.f;  // a split without tiles contributes nothing
      } else {
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
              if (direct) {
                const float l = l_run[h];
                orow[h * 512 + d] = l > 0.f ? o[hh] / l : 0.f;
              } else {
                orow[h * 512 + d] = o[hh];
              }
            }
          }
        }
      }
      if (st < 64) {
        if (direct) {
          if (lse) {
            const float l = l_run[st];
            lse[(long long)i * 64 + st] = l > 0.f ? (m_use[st] + log2f(l)) * 0.69314718055994531f : -INFINITY;
          }
        } else {
          orow[64 * 512 + st] = m_use[st];
          orow[64 * 512 + 64 + st] = l_run[st];
        }
      }
    }
  }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) {
    __syncwarp();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merge the splits of each query row: with M = max_s m_s,
//   o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  lse = (M + log2 of the denominator) * ln 2.
// One warp per (row, head, 128 latent dims): lane L owns dims 4 L .. 4 L + 3 and
// has every split's float4 load in flight before the weights are known.
constexpr int kCombineThreads = 256;
constexpr int kCombineMaxSplits = 16;
__global__ void __launch_bounds__(kCombineThreads) sparse_mla_combine_kernel(const float* __restrict__ part,
                                                                             int splits, float* __restrict__ o_lat,
                                                                             float* __restrict__ lse) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item = blockIdx.x * (kCombineThreads / 32) + warp;  // (row, head, quarter): the grid covers T x 256
  const int i = item >> 8, h = (item >> 2) & 63, qd = item & 3;
  const float* p = part + (long long)i * splits * kPartFloats;
  const int d = 128 * qd + 4 * lane;
  float4 x[kCombineMaxSplits];
#pragma unroll
  for (int s = 0; s < kCombineMaxSplits; ++s)
    if (s < splits) x[s] = *reinterpret_cast<const float4*>(p + (long long)s * kPartFloats + h * 512 + d);
  const float ms = lane < splits ? p[(long long)lane * kPartFloats + 64 * 512 + h] : -INFINITY;
  const float ls = lane < splits ? p[(long long)lane * kPartFloats + 64 * 512 + 64 + h] : 0.f;
  float M = ms;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmax_(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float w = (lane < splits && M > -INFINITY) ? fast_exp2(ms - M) : 0.f;
  float den = w * ls;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int s = 0; s < kCombineMaxSplits; ++s) {
    const float ws = __shfl_sync(0xffffffffu, w, s);
    if (s < splits) {
      acc.x = fmaf(ws, x[s].x, acc.x);
      acc.y = fmaf(ws, x[s].y, acc.y);
      acc.z = fmaf(ws, x[s].z, acc.z);
      acc.w = fmaf(ws, x[s].w, acc.w);
    }
  }
  *reinterpret_cast<float4*>(o_lat + ((long long)i * 64 + h) * 512 + d) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lse && qd == 0 && lane == 0) lse[(long long)i * 64 + h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace

// Splits per query row: enough CTAs to cover the SMs, at most one per 128-key
// tile and at most kMaxSplits; `ws_bytes` bounds them too.
constexpr int kMaxSplits = 16;
inline size_t sparse_mla_part_bytes(int T, int splits) { return size_t(T) * splits * kPartFloats * 4; }
inline int sparse_mla_ws_splits(int T, int topk) {
  const int ntiles = (topk + kTileKeys - 1) / kTileKeys;
  int s = T > 0 ? 320 / T : 1;
  return s < 1 ? 1 : (s > kMaxSplits ? kMaxSplits : (s > ntiles ? ntiles : s));
}

cudaError_t prepare_sparse_mla() {
  static_assert(kSmemAlloc <= 232448, "sparse MLA shared memory exceeds the per-CTA limit");
  return cudaFuncSetAttribute(sparse_mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
}

cudaError_t launch_sparse_mla(const MlaLaunch& p, const CUtensorMap& tmap_q) {
  if (p.T <= 0) return cudaSuccess;
  const float scale_log2 = p.scale * 1.4426950408889634f;
  const int ntiles = (p.topk + kTileKeys - 1) / kTileKeys;
  int splits = p.sm_count > 0 ? p.sm_count / p.T : 1;
  splits = splits < 1 ? 1 : (splits > kMaxSplits ? kMaxSplits : (splits > ntiles ? ntiles : splits));
  while (splits > 1 && (p.part == nullptr || sparse_mla_part_bytes(p.T, splits) > p.part_bytes)) --splits;
  const int per = (ntiles + splits - 1) / splits;
  splits = (ntiles + per - 1) / per;  // no split without tiles
  if (int64_t(p.T) * splits > INT32_MAX) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(sparse_mla_kernel, dim3(unsigned(p.T * splits)), dim3(kMlaThreads), kSmemAlloc, p.stream, 1,
                             p.kv, tmap_q, p.cache_rows, p.kv_start, p.idx, p.topk, scale_log2, p.o_lat, p.lse, splits,
                             per, p.part, WaitLimit{p.wait_ns});
  if (e != cudaSuccess || splits == 1) return e;
  static_assert(kMaxSplits <= kCombineMaxSplits, "the merge holds every split's load");
  return launch_pdl(sparse_mla_combine_kernel, dim3(unsigned(p.T) * (256u / (kCombineThreads / 32))),
                    dim3(kCombineThreads), 0, p.stream, 1, p.part, splits, p.o_lat, p.lse);
}

}  // namespace dsa
