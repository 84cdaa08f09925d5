// Reference oracle for the DSA sparse-attention step — TEST INFRASTRUCTURE ONLY.
//
// Plain, slow, fp64 C++ written from the method's definition.  Only the test
// suite, the package's smoke check and the benchmark's CPU-baseline leg may
// load this library.  It shares no code, header or constant with the CUDA
// path; the fixed dimensions below are restated here on purpose.
//
// Sources (pages on the method; the page title and section are cited):
//  * "2026 LLM architecture overview (2): DSA and MoE of GLM 5 / DSV3.2" (nlpx.cn), section 2.1 config table:
//    index_n_heads 32, index_head_dim 128, num_attention_heads 64,
//    kv_lora_rank 512, qk_rope_head_dim 64, qk_head_dim 256, index_topk 2048.
//  * same page, section 2.2: the lightning indexer scores each query against
//    every history position, is used only for ranking, and a top-k selector
//    keeps the index_topk best positions for the real attention.
//  * "From a trillion dot products to two thousand: how DSA breaks N^2" (clawlihai.cn), "DSA full flow": stage one is
//    the low-dimensional indexer dot product over all history and a top-2048;
//    stage two is full Q.K, softmax and the V mix over those 2048 only.
//  * The score form I[t,s] = sum_h w[t,h] * (q_I[t,h] . k_I[s]) with one key per
//    position shared by the heads, the latent (absorbed) attention score
//    (q_lat.c_kv + q_rope.k_rope)/sqrt(256), and o_lat = sum_j p_j c_kv[s_j]
//    are the problem statement's; the pages print no formula.
//
// Readings where the pages are silent:
//  * causality: query t sees positions 0..t (itself included), so the row has
//    n_vis = t+1 candidates and keeps min(topk, n_vis) of them;
//  * ties in the indexer score go to the lower position;
//  * the selected positions are reported in ascending order, padded with -1;
//  * all tensor inputs are bf16, widened exactly to double here.
//
// Every function takes `nthreads` and splits query rows across std::threads.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

const int kIdxHeads = 32;   // index_n_heads
const int kIdxDim = 128;    // index_head_dim
const int kHeads = 64;      // num_attention_heads
const int kLatent = 512;    // kv_lora_rank
const int kRope = 64;       // qk_rope_head_dim
const int kRow = kLatent + kRope;  // one latent-cache row

double widen_bf16(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

template <class F>
void for_rows(int T, int nthreads, F f) {
  if (nthreads <= 1 || T <= 1) {
    for (int i = 0; i < T; ++i) f(i);
    return;
  }
  int n = std::min(nthreads, T);
  std::vector<std::thread> pool;
  for (int k = 0; k < n; ++k)
    pool.emplace_back([&, k] {
      for (int i = k; i < T; i += n) f(i);
    });
  for (auto& t : pool) t.join();
}

// Indexer score of one query row against positions 0..n-1 of its sequence:
// I[s] = sum over the 32 heads of w[h] * (q_I[h] . k_I[s]).
void row_scores(const uint16_t* qI, const uint16_t* w, const uint16_t* kI_seq, int64_t n,
                double* out) {
  std::vector<double> q(kIdxHeads * kIdxDim), wh(kIdxHeads);
  for (int i = 0; i < kIdxHeads * kIdxDim; ++i) q[i] = widen_bf16(qI[i]);
  for (int h = 0; h < kIdxHeads; ++h) wh[h] = widen_bf16(w[h]);
  std::vector<double> k(kIdxDim);
  for (int64_t s = 0; s < n; ++s) {
    for (int d = 0; d < kIdxDim; ++d) k[d] = widen_bf16(kI_seq[s * kIdxDim + d]);
    double total = 0.0;
    for (int h = 0; h < kIdxHeads; ++h) {
      double dot = 0.0;
      for (int d = 0; d < kIdxDim; ++d) dot += q[h * kIdxDim + d] * k[d];
      total += wh[h] * dot;
    }
    out[s] = total;
  }
}

// Top-k of one row under the total order (score descending, position ascending);
// writes the kept positions in ascending order and pads with -1.
void row_topk(const double* score, int64_t n, int topk, int32_t* idx) {
  int64_t keep = std::min<int64_t>(topk, n);
  std::vector<int64_t> pos(n);
  for (int64_t s = 0; s < n; ++s) pos[s] = s;
  auto better = [score](int64_t a, int64_t b) {
    if (score[a] != score[b]) return score[a] > score[b];
    return a < b;
  };
  if (keep < n) std::nth_element(pos.begin(), pos.begin() + keep, pos.end(), better);
  std::sort(pos.begin(), pos.begin() + keep);
  for (int64_t j = 0; j < keep; ++j) idx[j] = static_cast<int32_t>(pos[j]);
  for (int64_t j = keep; j < topk; ++j) idx[j] = -1;
}

// Latent-form attention of one query over its selected cache rows.
// score_j = scale * (q_lat . c_kv[s_j] + q_rope . k_rope[s_j]);
// p = softmax over the selected j; o_lat = sum_j p_j c_kv[s_j]; lse = log sum_j exp(score_j).
// Slots holding -1 are not part of the set.  An empty set gives o = 0, lse = -inf.
void row_attention(const uint16_t* q, const uint16_t* kv_seq, const int32_t* idx, int topk,
                   double scale, double* o, double* lse) {
  std::vector<int32_t> sel;
  for (int j = 0; j < topk; ++j)
    if (idx[j] >= 0) sel.push_back(idx[j]);
  const size_t m = sel.size();
  std::vector<double> row(m * kRow);
  for (size_t j = 0; j < m; ++j)
    for (int d = 0; d < kRow; ++d) row[j * kRow + d] = widen_bf16(kv_seq[int64_t(sel[j]) * kRow + d]);
  std::vector<double> qh(kRow), sc(m);
  for (int h = 0; h < kHeads; ++h) {
    for (int d = 0; d < kRow; ++d) qh[d] = widen_bf16(q[h * kRow + d]);
    double* oh = o + int64_t(h) * kLatent;
    if (m == 0) {
      for (int d = 0; d < kLatent; ++d) oh[d] = 0.0;
      lse[h] = -std::numeric_limits<double>::infinity();
      continue;
    }
    double mx = -std::numeric_limits<double>::infinity();
    for (size_t j = 0; j < m; ++j) {
      const double* r = &row[j * kRow];
      double nope = 0.0, rope = 0.0;
      for (int d = 0; d < kLatent; ++d) nope += qh[d] * r[d];
      for (int d = 0; d < kRope; ++d) rope += qh[kLatent + d] * r[kLatent + d];
      sc[j] = (nope + rope) * scale;
      mx = std::max(mx, sc[j]);
    }
    double l = 0.0;
    for (size_t j = 0; j < m; ++j) {
      sc[j] = std::exp(sc[j] - mx);
      l += sc[j];
    }
    for (int d = 0; d < kLatent; ++d) oh[d] = 0.0;
    for (size_t j = 0; j < m; ++j) {
      const double p = sc[j] / l;
      const double* r = &row[j * kRow];
      for (int d = 0; d < kLatent; ++d) oh[d] += p * r[d];
    }
    lse[h] = mx + std::log(l);
  }
}

}  // namespace

extern "C" {

int oracle_dims(int* out6) {
  out6[0] = kIdxHeads;
  out6[1] = kIdxDim;
  out6[2] = kHeads;
  out6[3] = kLatent;
  out6[4] = kRope;
  out6[5] = kRow;
  return 6;
}

// scores[i, s] for s < n_vis[i]; entries at s >= n_vis[i] are left untouched.
void oracle_indexer_scores(const uint16_t* q_I, const uint16_t* w, const uint16_t* k_I,
                           const int64_t* kv_start, const int32_t* n_vis, int T, int64_t score_ld,
                           double* scores, int nthreads) {
  for_rows(T, nthreads, [&](int i) {
    row_scores(q_I + int64_t(i) * kIdxHeads * kIdxDim, w + int64_t(i) * kIdxHeads,
               k_I + kv_start[i] * kIdxDim, n_vis[i], scores + int64_t(i) * score_ld);
  });
}

void oracle_topk(const double* scores, int64_t score_ld, const int32_t* n_vis, int T, int topk,
                 int32_t* idx, int nthreads) {
  for_rows(T, nthreads, [&](int i) {
    row_topk(scores + int64_t(i) * score_ld, n_vis[i], topk, idx + int64_t(i) * topk);
  });
}

void oracle_sparse_mla(const uint16_t* q, const uint16_t* kv, const int64_t* kv_start,
                       const int32_t* idx, int T, int topk, double scale, double* o_lat,
                       double* lse, int nthreads) {
  for_rows(T, nthreads, [&](int i) {
    row_attention(q + int64_t(i) * kHeads * kRow, kv + kv_start[i] * kRow,
                  idx + int64_t(i) * topk, topk, scale, o_lat + int64_t(i) * kHeads * kLatent,
                  lse + int64_t(i) * kHeads);
  });
}

// The whole step for each row: scores -> top-k -> attention, one row at a time
// (no T x n_vis score matrix is held).  idx_out may be null.
void oracle_forward(const uint16_t* q_I, const uint16_t* w, const uint16_t* k_I, const uint16_t* q,
                    const uint16_t* kv, const int64_t* kv_start, const int32_t* n_vis, int T,
                    int topk, double scale, double* o_lat, double* lse, int32_t* idx_out,
                    int nthreads) {
  for_rows(T, nthreads, [&](int i) {
    std::vector<double> sc(n_vis[i]);
    std::vector<int32_t> idx(topk);
    row_scores(q_I + int64_t(i) * kIdxHeads * kIdxDim, w + int64_t(i) * kIdxHeads,
               k_I + kv_start[i] * kIdxDim, n_vis[i], sc.data());
    row_topk(sc.data(), n_vis[i], topk, idx.data());
    row_attention(q + int64_t(i) * kHeads * kRow, kv + kv_start[i] * kRow, idx.data(), topk,
                  scale, o_lat + int64_t(i) * kHeads * kLatent, lse + int64_t(i) * kHeads);
    if (idx_out) std::copy(idx.begin(), idx.end(), idx_out + int64_t(i) * topk);
  });
}

}  // extern "C"
