// Lightning-indexer scores on the 5th-generation tensor cores.
//
//   scores[i, s] = sum_{h<32} w[i,h] * (q_I[i,h,:] . k_I[kv_start[i]+s, :])
//
// ("2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2", section 2.2: a light scorer of every
// query against all history, 32 heads x 128 dims; the per-head weighting and
// head sum are the problem statement's.)
//
// Swap-AB formulation: one tcgen05.mma of M = 128 keys (TMEM lanes) x
// N = 32 * nq (heads x queries of one query tile) x K = 128 produces every
// head's dot product for 128 keys and up to 8 queries that share the
// sequence.  Keys arrive by TMA (two 64-column boxes, 128-byte swizzle) into
// a STAGES-deep ring; the query tile's q_I sits in its own buffer.  In the
// epilogue a warp reads its 32 key rows x 32 head columns per query with the
// 16x256b TMEM shape, so each lane sees 8 of the 32 heads (for 4 keys): the
// lane keeps those 8 weights of each of its queries in registers for the
// whole tile, weights and sums its 8 heads, and a 2-step shuffle
// reduce-scatter over the 4 lanes that share a key row finishes the head sum
// (one key per lane).  No weight is re-read from shared memory per key unit,
// which leaves the shared-memory pipe to the tensor core's operand reads.
//
// Warp roles: warp 0 = TMA producer, warp 1 = TMEM allocator and MMA issuer,
// warps 2.. = epilogue, P warps per TMEM lane quarter (P = 4 for the 8-query
// tile, else 2), warp part p taking queries p, p + P, ...  Each warp works
// through its share of a unit serially (TMEM load, head sum, store or filter),
// so that share, not the tensor core, sets the pace unless it is small: four
// warps per quarter keep it at two queries.  Persistent grid.
//
// Streamed selection (STREAM): no score is written.  Each score above its
// query's filter threshold goes, with its position, into the query's
// candidate buffer (workspace, kStreamCap entries).  A long tile first scores
// kSampleUnits key units spread over its range and seeds every threshold from
// them; every kCheckUnits units a buffer that could overflow is cut to its
// exact top-k and its threshold raised to the k-th score.  The exact top-k of
// the final buffers is taken afterwards by launch_stream_select; rows whose
// seeded filter let too few keys through are swept again unseeded first.
#pragma once
#include <cuda.h>

#include "block_scan.cuh"
#include "dsa.h"
#include "group_select.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kKeysPerUnit = 128;
constexpr int kStageBytes = kKeysPerUnit * 128 * 2;  // 32 KB: 128 keys x 128 dims bf16
constexpr int kHalfKeyBytes = kStageBytes / 2;       // one 64-column box
constexpr int kQRowsPerQuery = 32;                   // heads
constexpr int kQBoxBytes = kQRowsPerQuery * 64 * 2;  // 4 KB: one query, one 64-column half

// ------------------------------------------------------------------ plan kernel
__global__ void __launch_bounds__(1024) indexer_plan_kernel(const int64_t* __restrict__ kv_start,
                                                            const int32_t* __restrict__ n_vis, int T, int qmax,
                                                            int64_t score_ld, int64_t cache_rows,
                                                            PlanHeader* __restrict__ hdr,
                                                            PlanTile* __restrict__ tiles) {
  __shared__ int sc_i[33];
  __shared__ long long sc_l[33];
  __shared__ int carry_seg_s;
  const int tid = threadIdx.x;
  pdl_wait();  // inputs and the plan buffer may belong to the previous kernel
  pdl_trigger();
  for (int i = tid; i < T; i += blockDim.x) {
    PlanTile z;
    z.q0 = 0;
    z.nq = 0;
    z.units = 0;
    z.pad = 0;
    z.kv_start = 0;
    z.unit_begin = 0;
    tiles[i] = z;
  }
  __syncthreads();

  auto row_ok = [&](int i, long long& ks, int& nv) {
    ks = kv_start[i];
    nv = n_vis[i];
    return nv >= 1 && nv <= score_ld && ks >= 0 && ks + nv <= cache_rows;
  };

  int carry_seg = -1, carry_tiles = 0;
  for (int base = 0; base < T; base += blockDim.x) {
    const int i = base + tid;
    const bool in = i < T;
    long long ks = 0;
    int nv = 0;
    bool ok = false, head = false;
    if (in) {
      ok = row_ok(i, ks, nv);
      if (!ok) raise_status(kStatusBadRow);
      if (i == 0) {
        head = true;
      } else {
        long long ksp;
        int nvp;
        bool okp = row_ok(i - 1, ksp, nvp);
        head = !ok || !okp || ks != ksp;
      }
    }
    int seg = block_inclusive_max<int>(head ? i : -1, sc_i, -1);
    seg = seg > carry_seg ? seg : carry_seg;
    bool tstart = false;
    int q0 = 0;
    if (in) {
      q0 = seg + ((i - seg) / qmax) * qmax;
      tstart = (q0 == i);
    }
    int total = 0;
    int excl = block_exclusive_sum<int>(tstart ? 1 : 0, sc_i, &total);
    if (in) {
      const int tile = carry_tiles + excl - (tstart ? 0 : 1);
      if (tstart) {
        tiles[tile].q0 = i;
        tiles[tile].kv_start = ks;
      }
      atomicMax(&tiles[tile].nq, i - q0 + 1);
      atomicMax(&tiles[tile].units, ok ? (nv + kKeysPerUnit - 1) / kKeysPerUnit : 0);
    }
    const int last = (T - 1 - base) < int(blockDim.x - 1) ? (T - 1 - base) : int(blockDim.x - 1);
    if (tid == last) carry_seg_s = seg;
    __syncthreads();
    carry_seg = carry_seg_s;
    carry_tiles += total;
    __syncthreads();
  }
  __threadfence_block();
  __syncthreads();

  const int n_tiles = carry_tiles;
  long long carry = 0;
  for (int base = 0; base < n_tiles; base += blockDim.x) {
    const int j = base + tid;
    long long u = j < n_tiles ? (long long)tiles[j].units : 0;
    long long total = 0;
    long long ex = block_exclusive_sum<long long>(u, sc_l, &total);
    if (j < n_tiles) tiles[j].unit_begin = carry + ex;
    carry += total;
  }
  if (tid == 0) {
    hdr->total_units = carry;
    hdr->n_tiles = n_tiles;
  }
}

// Plan of the redo sweep: one tile per query listed in redo[1 .. redo[0]].
__global__ void __launch_bounds__(1024) indexer_redo_plan_kernel(const int* __restrict__ redo,
                                                                 const int64_t* __restrict__ kv_start,
                                                                 const int32_t* __restrict__ n_vis,
                                                                 PlanHeader* __restrict__ hdr,
                                                                 PlanTile* __restrict__ tiles) {
  __shared__ long long sc_l[33];
  pdl_wait();
  pdl_trigger();
  const int n = redo[0];
  long long carry = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int j = base + threadIdx.x;
    long long u = 0;
    PlanTile t{};
    if (j < n) {
      const int q = redo[1 + j];
      t.q0 = q;
      t.nq = 1;
      t.units = (n_vis[q] + kKeysPerUnit - 1) / kKeysPerUnit;
      t.kv_start = kv_start[q];
      u = t.units;
    }
    long long total = 0;
    const long long ex = block_exclusive_sum<long long>(u, sc_l, &total);
    if (j < n) {
      t.unit_begin = carry + ex;
      tiles[j] = t;
    }
    carry += total;
  }
  if (threadIdx.x == 0) {
    hdr->total_units = carry;
    hdr->n_tiles = n;
  }
}

// ------------------------------------------------------------------ unit iterator
// Every role of the main kernel walks the same sequence of (query tile, key tile).
struct UnitIter {
  const PlanTile* tiles;
  int n_tiles;
  int sweep;
  int samples = 0;  // sample units ahead of a long tile's sweep (wave sweep only)
  int tile;
  int kt;           // step within the tile: -ns .. -1 sample units, then 0 .. units-1
  int ns;           // this tile's sample units
  long long left;   // units left (split sweep)
  PlanTile cur;

  __device__ bool load_tile(int j) {
    while (j < n_tiles && tiles[j].units == 0) j += (sweep == kSweepWave ? int(gridDim.x) : 1);
    if (j >= n_tiles) return false;
    tile = j;
    cur = tiles[j];
    ns = (samples > 0 && cur.units >= kSampleMinUnits) ? samples : 0;
    return true;
  }
  // key unit of the current step; sample unit i of ns is unit i * units / ns
  __device__ int unit() const { return kt >= 0 ? kt : int((long long)(kt + ns) * cur.units / ns); }
  __device__ bool begin(const PlanHeader* hdr, const PlanTile* t) {
    tiles = t;
    n_tiles = hdr->n_tiles;
    const long long U = hdr->total_units;
    kt = 0;
    ns = 0;
    if (sweep == kSweepWave) {
      left = 1;
      if (!load_tile(int(blockIdx.x))) return false;
      kt = -ns;
      return true;
    }
    const long long G = gridDim.x;
    const long long b = U * (long long)blockIdx.x / G, e = U * (long long)(blockIdx.x + 1) / G;
    left = e - b;
    if (left <= 0) return false;
    // last tile whose unit_begin <= b
    int lo = 0, hi = n_tiles - 1;
    while (lo < hi) {
      int mid = (lo + hi + 1) >> 1;
      if (tiles[mid].unit_begin <= b) lo = mid;
      else hi = mid - 1;
    }
    if (!load_tile(lo)) return false;
    kt = int(b - cur.unit_begin);
    return true;
  }
  __device__ bool next() {
    ++kt;
    if (sweep != kSweepWave) {
      if (--left <= 0) return false;
    }
    if (kt < cur.units) return true;
    if (!load_tile(tile + (sweep == kSweepWave ? int(gridDim.x) : 1))) return false;
    kt = -ns;
    return true;
  }
};

// ------------------------------------------------------------------ main kernel
// Epilogue warps of a tile of QMAX queries (a multiple of 4: whole lane quarters).
template <int QMAX>
__host__ __device__ constexpr int epi_warps() {
  return QMAX == 8 ? 16 : 8;
}
template <int QMAX>
__host__ __device__ constexpr int idx_threads() {
  return 64 + 32 * epi_warps<QMAX>();
}
constexpr int kCheckUnits = 32;  // streaming selection: units between candidate-buffer checks
static_assert(kStreamCap - DSA_MAX_TOPK >= kCheckUnits * kKeysPerUnit,
              "a cut buffer must take every key of one check interval");

template <int QMAX, int STAGES, int QBUF, bool STREAM>
struct IdxSmem {
  static constexpr int kQBufBytes = QMAX * 2 * kQBoxBytes;  // two halves
  static constexpr int kKeysOff = 0;
  static constexpr int kQOff = STAGES * kStageBytes;
  static constexpr int kWOff = kQOff + QBUF * kQBufBytes;             // float w[QMAX*32]
  static constexpr int kNvOff = kWOff + QMAX * 32 * 4;                // int n_vis[QMAX]
  // streaming selection state: thresholds, counts, scan scratch, histogram, sort buffer
  static constexpr int kThrOff = (kNvOff + QMAX * 4 + 15) & ~15;      // long long thr[QMAX]
  static constexpr int kCntOff = kThrOff + QMAX * 8;                  // int cnt[QMAX]
  static constexpr int kSmpOff = kCntOff + QMAX * 4;                  // int seeded[QMAX]
  static constexpr int kGsOff = kSmpOff + QMAX * 4;                   // GroupShared
  static constexpr int kHistOff = (kGsOff + int(sizeof(GroupShared)) + 15) & ~15;  // uint32 hist[4096]
  static constexpr int kStreamEnd = STREAM ? kHistOff + 4096 * 4 : kNvOff + QMAX * 4;
  static constexpr int kBarOff = (kStreamEnd + 7) & ~7;
  static constexpr int kNumBars = 2 * STAGES + 2 * QBUF + 4 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;             // tmem slot, abort flag
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;                        // slack for 1 KB alignment
  static constexpr int kAccCols = 32 * QMAX;
  static constexpr int kTmemCols = (2 * kAccCols) <= 32 ? 32 : (2 * kAccCols);
};

template <int QMAX, int STAGES, int QBUF, bool STREAM>
__global__ void __launch_bounds__(idx_threads<QMAX>(), 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                   const uint16_t* __restrict__ w, const int32_t* __restrict__ n_vis,
                   const PlanHeader* __restrict__ hdr, const PlanTile* __restrict__ tiles, float* __restrict__ scores,
                   int64_t score_ld, int sweep, StreamOut so, WaitLimit lim) {
  using L = IdxSmem<QMAX, STAGES, QBUF, STREAM>;
  constexpr int EPI = epi_warps<QMAX>();  // epilogue warps
  constexpr int P = EPI / 4;              // epilogue warps per TMEM lane quarter
  constexpr int J = (QMAX + P - 1) / P;   // queries per epilogue warp (at most)
  extern __shared__ uint8_t smem_raw[];
  // 1 KB-aligned base by pointer arithmetic on the shared array (an integer round trip
  // would hide the shared address space and turn every access into a generic one)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  float* w_s = reinterpret_cast<float*>(smem + L::kWOff);
  int* nv_s = reinterpret_cast<int*>(smem + L::kNvOff);
  const uint32_t bar0 = sbase + L::kBarOff;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto qfull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + b); };
  auto qempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + QBUF + b); };
  auto afull_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * QBUF + b); };
  auto aempty_bar = [&](int b) { return bar0 + 8u * (2 * STAGES + 2 * QBUF + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 2 * QBUF + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < QBUF; ++b) {
      mbar_init(qfull_bar(b), 1);
      mbar_init(qempty_bar(b), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(afull_bar(b), 1);
      mbar_init(aempty_bar(b), EPI);  // one arrival per epilogue warp
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // everything above touched shared memory and TMEM only

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      UnitIter it;
      it.sweep = sweep;
      it.samples = STREAM ? so.sample_units : 0;
      int stage = 0, qb = -1, prev_tile = -1;
      uint32_t phase = 0;
      uint32_t qphase[QBUF];
      for (int b = 0; b < QBUF; ++b) qphase[b] = 0;
      int issued[STAGES], q_issued[QBUF];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      for (int b = 0; b < QBUF; ++b) q_issued[b] = 0;
      bool ok = it.begin(hdr, tiles);
      while (ok) {
        if (it.tile != prev_tile) {
          qb = (qb + 1) % QBUF;
          if (!mbar_wait(qempty_bar(qb), qphase[qb] ^ 1u, lim, abort_flag)) break;
          const int nq = it.cur.nq;
          mbar_arrive_expect_tx(qfull_bar(qb), uint32_t(nq) * 2u * kQBoxBytes);
          const uint32_t qdst = sbase + L::kQOff + qb * L::kQBufBytes;
          for (int qi = 0; qi < nq; ++qi) {
            const int y = (it.cur.q0 + qi) * kQRowsPerQuery;
            tma_load_2d(qdst + qi * kQBoxBytes, &tmap_q, qfull_bar(qb), 0, y);
            tma_load_2d(qdst + QMAX * kQBoxBytes + qi * kQBoxBytes, &tmap_q, qfull_bar(qb), 64, y);
          }
          qphase[qb] ^= 1u;
          ++q_issued[qb];
          prev_tile = it.tile;
        }
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, lim, abort_flag)) break;
        mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
        const int y = int(it.cur.kv_start + (long long)it.unit() * kKeysPerUnit);
        const uint32_t kdst = sbase + L::kKeysOff + stage * kStageBytes;
        tma_load_2d(kdst, &tmap_k, full_bar(stage), 0, y);
        tma_load_2d(kdst + kHalfKeyBytes, &tmap_k, full_bar(stage), 64, y);
        ++issued[stage];
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        ok = it.next();
      }
      // Drain: every key stage and query buffer we loaded must have landed before
      // the CTA exits (on an abort the MMA warp may not have consumed them).
      for (int s = 0; s < STAGES; ++s)
        if (issued[s] > 0) mbar_drain(full_bar(s), uint32_t((issued[s] - 1) & 1));
      for (int b = 0; b < QBUF; ++b)
        if (q_issued[b] > 0) mbar_drain(qfull_bar(b), uint32_t((q_issued[b] - 1) & 1));
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      UnitIter it;
      it.sweep = sweep;
      it.samples = STREAM ? so.sample_units : 0;
      int stage = 0, qb = -1, prev_tile = -1, ab = 0;
      uint32_t phase = 0, aphase = 0;
      uint32_t qphase[QBUF];
      for (int b = 0; b < QBUF; ++b) qphase[b] = 0;
      bool ok = it.begin(hdr, tiles);
      while (ok) {
        if (it.tile != prev_tile) {
          if (qb >= 0) mma_commit(qempty_bar(qb));  // previous query buffer free once its MMAs finish
          qb = (qb + 1) % QBUF;
          if (!mbar_wait(qfull_bar(qb), qphase[qb], lim, abort_flag)) break;
          qphase[qb] ^= 1u;
          prev_tile = it.tile;
        }
        if (!mbar_wait(aempty_bar(ab), aphase ^ 1u, lim, abort_flag)) break;
        if (!mbar_wait(full_bar(stage), phase, lim, abort_flag)) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16(128, 32 * it.cur.nq, 0, 0);
        const uint32_t kaddr = sbase + L::kKeysOff + stage * kStageBytes;
        const uint32_t qaddr = sbase + L::kQOff + qb * L::kQBufBytes;
        const uint32_t d_tmem = tmem_base + uint32_t(ab * L::kAccCols);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t koff = uint32_t((k >> 2) * kHalfKeyBytes + (k & 3) * 32);
          const uint32_t qoff = uint32_t((k >> 2) * QMAX * kQBoxBytes + (k & 3) * 32);
          const uint64_t ad = smem_desc(kaddr + koff, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(qaddr + qoff, 16, 1024, kSwizzle128B);
          mma_bf16_ss(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(empty_bar(stage));
        mma_commit(afull_bar(ab));
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        if (++ab == 2) {
          ab = 0;
          aphase ^= 1u;
        }
        ok = it.next();
      }
      // Drain: wait until every MMA issued above has completed (also after an
      // abort: TMEM is released only once no MMA can still write it).
      mma_commit(drain_bar);
      mbar_drain(drain_bar, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 2 .. 1 + EPI)
    const int quarter = warp & 3;         // TMEM lane quarter this warp may access
    const int part = (warp - 2) >> 2;     // queries part, part + P, part + 2P, ...
    // after the head reduce-scatter lane t holds key row t / 4 + 8 (t % 4) of the quarter
    const int row = quarter * 32 + (lane >> 2) + 8 * (lane & 3);
    const int hc = 2 * (lane & 3);        // this lane's heads: 8i + hc + {0, 1}, i < 4
    const int et = threadIdx.x - 64;      // 0 .. 32 * EPI - 1
    long long* thr_s = reinterpret_cast<long long*>(smem + L::kThrOff);
    int* cnt_s = reinterpret_cast<int*>(smem + L::kCntOff);
    int* seeded_s = reinterpret_cast<int*>(smem + L::kSmpOff);
    GroupShared& gs = *reinterpret_cast<GroupShared*>(smem + L::kGsOff);
    uint32_t* hist = reinterpret_cast<uint32_t*>(smem + L::kHistOff);
    // Keep the topk best entries of query q's buffer (exact: ties at the cut go to the
    // lowest positions), move them to its front and raise its filter threshold.
    auto stream_shrink = [&](int q, int q0, const Group& g) {
      const long long ro = (long long)(q0 + q) * so.cap;
      const int m = min(cnt_s[q], so.cap);
      if (m <= so.topk) return;
      const uint32_t* ck = so.cand_key + ro;
      int32_t* cp = so.cand_pos + ro;
      const Rule r = group_radix_select(m, so.topk, hist, gs, g, [&](int j) { return ck[j]; },
                                        [](int) { return true; });
      long long cut = 0;  // among keys == r.thr keep positions p with ~p >= cut
      if (r.keep_eq > 0 && r.keep_eq < r.count_eq) {  // some tied keys must go: lowest positions stay
        const Rule rp = group_radix_select(
            m, r.keep_eq, hist, gs, g, [&](int j) { return ~uint32_t(cp[j]); },
            [&](int j) { return (long long)ck[j] == r.thr; });
        cut = rp.keep_eq > 0 ? rp.thr : rp.thr + 1;
      }
      const int kept = group_compact(
          m, gs, g, [&](int j) { return make_uint2(ck[j], uint32_t(cp[j])); },
          [&](uint2 e) {
            const long long k = e.x;
            return k > r.thr || (r.keep_eq > 0 && k == r.thr && (long long)(~e.y) >= cut);
          },
          [&](int dst, uint2 e) {
            so.cand_key[ro + dst] = e.x;
            so.cand_pos[ro + dst] = int32_t(e.y);
          });
      if (g.tid == 0) {
        cnt_s[q] = kept;
        thr_s[q] = r.thr;
      }
      g.sync();
    };
    // After the sample units: start query q's filter at a threshold that about
    // (1 + 4 / sqrt(share)) x topk of its keys should pass, share being the
    // sample's expected part of its topk; the buffer is emptied (the main sweep
    // visits the sampled keys again).  Rows that fit the buffer keep every key.
    auto stream_seed = [&](int q, int q0, const Group& g) {
      const long long ro = (long long)(q0 + q) * so.cap;
      const int S = min(cnt_s[q], so.cap);
      const int n = nv_s[q];
      long long t = -1;
      int seeded = 0;
      if (n > so.cap && S > 0) {
        int r = 1;
        if (so.sample_mode != 2) {
          const float share = float(so.topk) * float(S) / float(n);
          r = int(ceilf(share + 4.0f * sqrtf(share))) + 8;
        }
        if (r < S) {
          const Rule rr = group_radix_select(S, r, hist, gs, g, [&](int j) { return so.cand_key[ro + j]; },
                                             [](int) { return true; });
          t = rr.keep_eq > 0 ? rr.thr - 1 : rr.thr;  // keys >= the r-th largest sample key pass
          seeded = 1;
        }
      }
      if (g.tid == 0) {
        thr_s[q] = t;
        cnt_s[q] = 0;
        seeded_s[q] = seeded;
      }
      g.sync();
    };
    // End of query q's sweep: hand its candidate count to the selection kernel
    // that runs after the sweeps (exact top-k of the buffer, written ascending).
    // A seeded filter that let fewer than min(topk, n) keys through (no cut
    // happened, or cnt would be >= topk) may have dropped some of the best: the
    // query goes on the redo list instead and is swept again unseeded.
    auto stream_finish = [&](int q, int q0) {
      if (et != 0) return;
      if (seeded_s[q] && cnt_s[q] < min(so.topk, nv_s[q])) so.redo[1 + atomicAdd(so.redo, 1)] = q0 + q;
      else so.cnt_out[q0 + q] = min(cnt_s[q], so.cap);
    };
    // This thread's queries are part + P j, j < J (slot j);
    // their visible lengths and filter thresholds live in registers, reloaded from
    // shared memory only where they change (tile start, seeding, buffer checks).
    int nv_r[J];
    long long thr_r[J];
    float wr[J][8];  // wr[j][2i + e] = w[query part + P j, head 8i + hc + e]
    auto refresh = [&]() {
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int q = part + P * j;
        nv_r[j] = q < QMAX ? nv_s[q] : 0;
        thr_r[j] = (STREAM && q < QMAX) ? thr_s[q] : -1;
      }
    };
    UnitIter it;
    it.sweep = sweep;
    it.samples = STREAM ? so.sample_units : 0;
    int prev_tile = -1, ab = 0;
    uint32_t aphase = 0;
    // A warp whose accumulator wait fails stops working but keeps walking the
    // same units, so it still takes every named barrier and group step the
    // other epilogue warps take (leaving the loop early could strand them).
    bool alive = true;
    bool ok = it.begin(hdr, tiles);
    while (ok) {
      const int nq = it.cur.nq;
      if (it.tile != prev_tile) {
        named_bar_sync(1, 32 * EPI);
        for (int e = et; e < nq * 32; e += 32 * EPI)
          w_s[e] = bf16_bits_to_float(w[(long long)it.cur.q0 * 32 + e]);
        if (et < QMAX) nv_s[et] = et < nq ? n_vis[it.cur.q0 + et] : 0;
        if constexpr (STREAM) {
          if (et < QMAX) {
            thr_s[et] = -1;  // nothing kept yet: every score passes
            cnt_s[et] = 0;
            seeded_s[et] = 0;
          }
        }
        named_bar_sync(1, 32 * EPI);
        refresh();
#pragma unroll
        for (int j = 0; j < J; ++j) {
          const int q = part + P * j;
#pragma unroll
          for (int e = 0; e < 8; ++e) wr[j][e] = q < nq ? w_s[q * 32 + 8 * (e >> 1) + hc + (e & 1)] : 0.f;
        }
        prev_tile = it.tile;
      }
      if (alive) alive = __all_sync(0xffffffffu, mbar_wait(afull_bar(ab), aphase, lim, abort_flag));
      tc_fence_after();
      const long long s = (long long)it.unit() * kKeysPerUnit + row;
      const uint32_t tbase = tmem_base + (uint32_t(quarter * 32) << 16) + uint32_t(ab * L::kAccCols);
      // score of (query qi, key s): written out, or offered to the query's candidate buffer
      // append the passing scores of query slot j (qi = part + P j) to its buffer
      auto append = [&](int j, uint32_t key, bool pass) {
        const int qi = part + P * j;
        const unsigned m = __ballot_sync(0xffffffffu, pass);
        if (m) {
          const int leader = __ffs(m) - 1;
          int base = 0;
          if (lane == leader) base = atomicAdd(&cnt_s[qi], __popc(m));
          base = __shfl_sync(0xffffffffu, base, leader);
          const int off = base + __popc(m & ((1u << lane) - 1u));
          if (pass && off < so.cap) {
            const long long ro = (long long)(it.cur.q0 + qi) * so.cap;
            so.cand_key[ro + off] = key;
            so.cand_pos[ro + off] = int(s);
          }
        }
      };
      // This warp's queries qi = part + P j, one TMEM wait each.
      // All scores are computed first and the accumulator is handed back to the
      // MMA warp before any is written or offered to a selection buffer.
      float sc[J];
#pragma unroll
      for (int j = 0; j < J; ++j) {
        const int qi = part + P * j;
        sc[j] = 0.f;
        if (alive && qi < nq) {  // warp-uniform
          float v[32];
          const uint32_t tq = tbase + uint32_t(qi * 32);
          tmem_ld16x256b_x4x2_sync(tq, tq + (16u << 16), v);
          // p[r]: this lane's 8 heads of key row (lane / 4) + 8r
          float p[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float* x = v + 16 * (r >> 1) + 2 * (r & 1);
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              acc = fmaf(wr[j][2 * i], x[4 * i], acc);
              acc = fmaf(wr[j][2 * i + 1], x[4 * i + 1], acc);
            }
            p[r] = acc;
          }
          // reduce-scatter over lanes t ^ 2, t ^ 1: lane t keeps key row t / 4 + 8 (t % 4)
          const bool b1 = (lane & 2) != 0, b0 = (lane & 1) != 0;
          float k0 = b1 ? p[2] : p[0], k1 = b1 ? p[3] : p[1];
          const float s0 = b1 ? p[0] : p[2], s1 = b1 ? p[1] : p[3];
          k0 += __shfl_xor_sync(0xffffffffu, s0, 2);
          k1 += __shfl_xor_sync(0xffffffffu, s1, 2);
          const float kk = b0 ? k1 : k0, ss = b0 ? k0 : k1;
          sc[j] = kk + __shfl_xor_sync(0xffffffffu, ss, 1);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (alive && lane == 0) mbar_arrive(aempty_bar(ab));
      if constexpr (!STREAM) {
#pragma unroll
        for (int j = 0; j < J; ++j)
          if (alive && s < nv_r[j]) scores[(long long)(it.cur.q0 + part + P * j) * score_ld + s] = sc[j];
      } else {
        // one vote for the common case that no score of the warp passes its filter
        uint32_t key[J];
        bool pass[J];
        bool any = false;
#pragma unroll
        for (int j = 0; j < J; ++j) {
          key[j] = float_order_key(sc[j]);
          pass[j] = alive && s < nv_r[j] && (long long)key[j] > thr_r[j];
          any = any || pass[j];
        }
        if (__any_sync(0xffffffffu, any)) {
#pragma unroll
          for (int j = 0; j < J; ++j)
            if (part + P * j < nq) append(j, key[j], pass[j]);
        }
      }
      if constexpr (STREAM) {
        const Group g{et, 32 * EPI, 1};
        if (it.kt < 0) {
          // the sample units fill at most kSampleUnits * 128 = cap entries; after
          // the last one, seed each query's threshold
          if (it.kt == -1) {
            g.sync();
            for (int q = 0; q < nq; ++q) stream_seed(q, it.cur.q0, g);
            refresh();
          }
        } else {
          // Every kCheckUnits units: shrink buffers that could overflow before the
          // next check (a query gains at most one entry per key); after the tile's
          // last unit, finish its queries.
          const bool last = it.kt == it.cur.units - 1;
          if (last || (it.kt % kCheckUnits) == kCheckUnits - 1) {
            g.sync();
            for (int q = 0; q < nq; ++q)
              if (cnt_s[q] > so.cap - kCheckUnits * kKeysPerUnit) stream_shrink(q, it.cur.q0, g);
            if (last)
              for (int q = 0; q < nq; ++q) stream_finish(q, it.cur.q0);
            refresh();
          }
        }
      }
      if (++ab == 2) {
        ab = 0;
        aphase ^= 1u;
      }
      ok = it.next();
    }
  }

  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, L::kTmemCols);
  }
}

template <int QMAX, int STAGES, int QBUF, bool STREAM>
cudaError_t set_smem_attr() {
  using L = IdxSmem<QMAX, STAGES, QBUF, STREAM>;
  static_assert(L::kAlloc <= 232448, "indexer shared memory exceeds the per-CTA limit");
  return cudaFuncSetAttribute(indexer_kernel<QMAX, STAGES, QBUF, STREAM>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
}

template <int QMAX, int STAGES, int QBUF, bool STREAM>
cudaError_t launch_main(const IndexerLaunch& p, const CUtensorMap& tk, const CUtensorMap& tq) {
  using L = IdxSmem<QMAX, STAGES, QBUF, STREAM>;
  auto* hdr = reinterpret_cast<const PlanHeader*>(p.plan);
  auto* tiles = reinterpret_cast<const PlanTile*>(reinterpret_cast<const uint8_t*>(p.plan) + sizeof(PlanHeader));
  return launch_pdl(indexer_kernel<QMAX, STAGES, QBUF, STREAM>, dim3(p.grid), dim3(idx_threads<QMAX>()), L::kAlloc,
                    p.stream, 1, tk, tq, p.w, p.n_vis, hdr, tiles, p.scores, p.score_ld, p.sweep, p.stream_out,
                    WaitLimit{p.wait_ns});
}

}  // namespace

cudaError_t prepare_indexer() {
  cudaError_t e;
  if ((e = set_smem_attr<1, 6, 2, false>()) != cudaSuccess) return e;
  if ((e = set_smem_attr<4, 4, 2, false>()) != cudaSuccess) return e;
  if ((e = set_smem_attr<8, 4, 1, false>()) != cudaSuccess) return e;
  if ((e = set_smem_attr<8, 4, 1, true>()) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_indexer(const IndexerLaunch& p, const CUtensorMap& tmap_k, const CUtensorMap& tmap_q) {
  if (p.T <= 0) return cudaSuccess;
  static_assert(kSampleUnits * kKeysPerUnit <= kStreamCap, "the sample fills at most the candidate buffer");
  if (p.streaming) {
    cudaError_t e0 = cudaMemsetAsync(p.stream_out.redo, 0, sizeof(int), p.stream);
    if (e0 == cudaSuccess) e0 = cudaMemsetAsync(p.stream_out.cnt_out, 0xFF, size_t(p.T) * 4, p.stream);
    if (e0 != cudaSuccess) return e0;
  }
  auto* hdr = reinterpret_cast<PlanHeader*>(p.plan);
  auto* tiles = reinterpret_cast<PlanTile*>(reinterpret_cast<uint8_t*>(p.plan) + sizeof(PlanHeader));
  cudaError_t e = launch_pdl(indexer_plan_kernel, dim3(1), dim3(1024), 0, p.stream, 1, p.kv_start, p.n_vis, p.T,
                             p.qmax, p.score_ld, p.cache_rows, hdr, tiles);
  if (e != cudaSuccess) return e;
  if (p.streaming) {
    if (p.qmax != 8 || p.sweep != kSweepWave) return cudaErrorInvalidValue;
    if ((e = launch_main<8, 4, 1, true>(p, tmap_k, tmap_q)) != cudaSuccess) return e;
    // queries whose seeded threshold let too few keys through: sweep them again,
    // unseeded (an empty list costs one short launch, no host round trip)
    if ((e = launch_pdl(indexer_redo_plan_kernel, dim3(1), dim3(1024), 0, p.stream, 1, p.stream_out.redo,
                        p.kv_start, p.n_vis, hdr, tiles)) != cudaSuccess)
      return e;
    IndexerLaunch p2 = p;
    p2.stream_out.sample_units = 0;
    return launch_main<8, 4, 1, true>(p2, tmap_k, tmap_q);
  }
  switch (p.qmax) {
    case 1: return launch_main<1, 6, 2, false>(p, tmap_k, tmap_q);
    case 4: return launch_main<4, 4, 2, false>(p, tmap_k, tmap_q);
    case 8: return launch_main<8, 4, 1, false>(p, tmap_k, tmap_q);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace dsa
