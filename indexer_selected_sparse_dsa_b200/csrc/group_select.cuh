// Selection helpers for a group of warps inside a warp-specialised CTA (the
// indexer's epilogue warps): scans, exact radix select, in-place compaction
// and a bitonic sort, synchronised with one named barrier instead of
// __syncthreads so the other roles of the CTA keep running.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

namespace {

struct Group {
  int tid;  // 0 .. n-1
  int n;    // threads in the group (a multiple of 32, <= 1024)
  int bar;  // named barrier id
  __device__ __forceinline__ void sync() const { named_bar_sync(bar, n); }
};

struct GroupShared {
  int scan[33];
  int sel_bin, sel_above, sel_count;
};

// Order-preserving 32-bit key of a float (-0 folded onto +0).
__device__ __forceinline__ uint32_t float_order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u << 1) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int group_exclusive_sum(int v, GroupShared& gs, int* total, const Group& g) {
  const int lane = g.tid & 31, w = g.tid >> 5, nw = g.n >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  if (lane == 31) gs.scan[w] = inc;
  g.sync();
  if (w == 0) {
    const int s = lane < nw ? gs.scan[lane] : 0;
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += t;
    }
    if (lane < nw) gs.scan[lane] = si - s;
    if (lane == nw - 1) gs.scan[32] = si;
  }
  g.sync();
  const int out = gs.scan[w] + inc - v;
  *total = gs.scan[32];
  g.sync();
  return out;
}

struct Rule {
  long long thr;  // keep key > thr ...
  int keep_eq;    // ... and the first keep_eq keys == thr (by the caller's tie order)
};

// Exact selection of the need-th largest key among the m entries with inc(j);
// key(j) returns a 32-bit order key.  hist holds >= 4096 words.
template <class Key, class Inc>
__device__ Rule group_radix_select(int m, int need, uint32_t* hist, GroupShared& gs, const Group& g, Key key,
                                   Inc inc) {
  uint32_t prefix = 0;
  int bits_done = 0;
  const int widths[3] = {12, 10, 10};
  for (int p = 0; p < 3; ++p) {
    const int w = widths[p];
    const int shift = 32 - bits_done - w;
    const int nb = 1 << w;
    for (int b = g.tid; b < nb; b += g.n) hist[b] = 0u;
    g.sync();
    for (int j = g.tid; j < m; j += g.n) {
      if (!inc(j)) continue;
      const uint32_t k = key(j);
      if (bits_done == 0 || (k >> (32 - bits_done)) == prefix) atomicAdd(&hist[(k >> shift) & uint32_t(nb - 1)], 1u);
    }
    g.sync();
    // bin where the count from the top first reaches `need`
    const int per = nb / g.n > 0 ? nb / g.n : 1;
    const int top = nb - 1 - g.tid * per;
    const bool owns = g.tid * per < nb;
    int local = 0;
    if (owns)
      for (int q = 0; q < per; ++q) local += int(hist[top - q]);
    int total = 0;
    const int ex = group_exclusive_sum(local, gs, &total, g);
    if (owns && ex < need && ex + local >= need) {
      int run = ex;
      for (int q = 0; q < per; ++q) {
        const int c = int(hist[top - q]);
        if (run + c >= need) {
          gs.sel_bin = top - q;
          gs.sel_above = run;
          gs.sel_count = c;
          break;
        }
        run += c;
      }
    }
    g.sync();
    prefix = (prefix << w) | uint32_t(gs.sel_bin);
    need -= gs.sel_above;
    bits_done += w;
    const bool whole = (gs.sel_count == need);
    g.sync();
    if (whole) return Rule{((long long)prefix << (32 - bits_done)) - 1, 0};
  }
  return Rule{(long long)prefix, need};
}

// In-place stable compaction: entry j (read with load(j)) is kept when keep(e);
// kept entries are written to the front with store(dst, e), dst <= j.  Every
// entry of a chunk is loaded into registers before any store of that chunk
// (the scan's barriers separate them).  Returns how many were kept.
template <class Load, class Keep, class Store>
__device__ int group_compact(int m, GroupShared& gs, const Group& g, Load load, Keep keep, Store store) {
  int written = 0;
  for (int base = 0; base < m; base += g.n) {
    const int j = base + g.tid;
    auto e = load(j < m ? j : 0);
    const bool k = j < m && keep(e);
    int tot = 0;
    const int o = written + group_exclusive_sum(k ? 1 : 0, gs, &tot, g);
    if (k) store(o, e);
    g.sync();
    written += tot;
  }
  return written;
}

// Ascending bitonic sort of buf[0, npow2) (npow2 a power of two).
__device__ void group_bitonic_sort(int* buf, int npow2, const Group& g) {
  for (int k = 2; k <= npow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = g.tid; i < npow2; i += g.n) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool asc = (i & k) == 0;
          const int a = buf[i], b = buf[ixj];
          if ((a > b) == asc) {
            buf[i] = b;
            buf[ixj] = a;
          }
        }
      }
      g.sync();
    }
  }
}

}  // namespace

}  // namespace dsa
