// Selection helpers for a group of warps inside a warp-specialised CTA (the
// indexer's epilogue warps): scans, exact radix select and in-place
// compaction, synchronised with one named barrier instead of __syncthreads so
// the other roles of the CTA keep running.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

namespace {

constexpr int kBatch = 8;  // entries per thread in flight in the selection loops

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
  int count_eq;   // how many entries have key == thr (when keep_eq > 0)
};

// Exact selection of the need-th largest key among the m entries with inc(j);
// key(j) returns a 32-bit order key.  The digits, from the top, are
// widths[0 .. npass - 1] bits wide (summing to 32); hist holds
// 1 << max(widths) words.
template <class Key, class Inc>
__device__ Rule group_radix_select_digits(int m, int need, uint32_t* hist, GroupShared& gs, const Group& g, Key key,
                                          Inc inc, const int* widths, int npass) {
  uint32_t prefix = 0;
  int bits_done = 0;
  for (int p = 0; p < npass; ++p) {
    const int w = widths[p];
    const int shift = 32 - bits_done - w;
    const int nb = 1 << w;
    for (int b = g.tid; b < nb; b += g.n) hist[b] = 0u;
    g.sync();
    // entries may sit in global memory: kBatch loads in flight per thread
    for (int j0 = g.tid; j0 < m; j0 += g.n * kBatch) {
      uint32_t kk[kBatch];
      bool in[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = j0 + u * g.n;
        in[u] = j < m && inc(j);
        kk[u] = in[u] ? key(j) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (in[u] && (bits_done == 0 || (kk[u] >> (32 - bits_done)) == prefix))
          atomicAdd(&hist[(kk[u] >> shift) & uint32_t(nb - 1)], 1u);
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
    const int count = gs.sel_count;
    g.sync();
    if (count == need) return Rule{((long long)prefix << (32 - bits_done)) - 1, 0, 0};
    if (p == npass - 1) return Rule{(long long)prefix, need, count};
  }
  return Rule{0, 0, 0};  // not reached
}

// The same with 12 + 10 + 10 bit digits (three passes; hist holds 4096 words).
template <class Key, class Inc>
__device__ Rule group_radix_select(int m, int need, uint32_t* hist, GroupShared& gs, const Group& g, Key key,
                                   Inc inc) {
  const int widths[3] = {12, 10, 10};
  return group_radix_select_digits(m, need, hist, gs, g, key, inc, widths, 3);
}

// In-place stable compaction: entry j (read with load(j)) is kept when keep(e);
// kept entries are written to the front with store(dst, e), dst <= j.  Each
// round covers kBatch consecutive entries per thread, all loaded into registers
// before any store of the round (the scan's barriers separate them).  Returns
// how many were kept.
template <class Load, class Keep, class Store>
__device__ int group_compact(int m, GroupShared& gs, const Group& g, Load load, Keep keep, Store store) {
  int written = 0;
  for (int base = 0; base < m; base += g.n * kBatch) {
    const int j0 = base + g.tid * kBatch;
    decltype(load(0)) e[kBatch];
    unsigned km = 0u;
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (j0 + u < m) {
        e[u] = load(j0 + u);
        if (keep(e[u])) km |= 1u << u;
      }
    int tot = 0;
    int o = written + group_exclusive_sum(__popc(km), gs, &tot, g);
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if ((km >> u) & 1u) store(o++, e[u]);
    g.sync();
    written += tot;
  }
  return written;
}

}  // namespace

}  // namespace dsa
