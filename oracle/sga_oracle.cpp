// SGA oracle: a plain, slow, fp64 CPU restatement of the Sparse Gated Attention
// (SGA) hot path.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the
// smoke check and by the CPU-baseline leg of the benchmark, never by the product
// path.  It shares no code, header or constant with the CUDA library.
//
// What it computes, step by step, with the passage each step follows:
//
//   Indexer (archdb "A.X K2", token-selection field: DSA-style indexer with 64
//   indexer heads of dim 128, ReLU-scored; indexer key width 128 per token):
//       score(t, s) = sum_j w[t,j] * max(0, sum_d q_idx[t,j,d] * k_idx[s,d])
//   for every causal past position s <= t.  The pages name the ingredients but
//   print no formula; this weighted sum of ReLU'd per-head dot products is the
//   stated DSA-style reading.  No scale, no bias.
//
//   Selection (same field: "top-2048 tokens per query"; arXiv abstract "A.X K2
//   Technical Report": each query reads only 2,048 positions):
//       keep the K positions with the largest score, ties going to the lower
//       position; if the query has t+1 <= K candidates keep all of them.
//       Output: ascending positions, padded with -1.
//
//   Attention (archdb "A.X K2" attention fields: MLA, 64 query heads, qk head
//   dim 192 = 128 nope + 64 rope, KV latent 512 + shared rope key 64), in the
//   absorbed (latent) form: per head h,
//       z_s = (q[h] . c_s) * scale            over the selected s (c_s: 576-wide row)
//       p   = softmax(z)
//       o[h]= sum_s p_s * c_s[0:Dv]           (Dv = 512: the latent part is the value)
//   with scale = 192^-0.5 (the qk head dim).
//
//   Gate (archdb "A.X K2" gate field: head-specific sigmoid gate on the
//   attention output before o_proj; nlp.com.ai "A.X K2 FP8": head-specific
//   output gating):
//       out[h] = o[h] / (1 + exp(-g[h]))      one scalar per (query, head)
//
// All arithmetic is in double.  Inputs are bf16 bit patterns (uint16) decoded
// exactly.  Threads split independent queries (and key ranges of one query in
// the indexer); no step is reordered or fused beyond the definitions above.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <utility>
#include <vector>

namespace {

double bf16_value(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

int pick_threads(int requested) {
  if (requested > 0) return requested;
  unsigned hc = std::thread::hardware_concurrency();
  return hc == 0 ? 1 : static_cast<int>(hc);
}

// Run body(i) for i in [0, n) on up to n_threads threads (static split).
template <class F>
void parallel_for(int64_t n, int n_threads, F body) {
  n_threads = static_cast<int>(std::min<int64_t>(std::max(1, n_threads), std::max<int64_t>(n, 1)));
  if (n_threads <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  for (int th = 0; th < n_threads; ++th) {
    pool.emplace_back([=]() {
      int64_t lo = n * th / n_threads, hi = n * (th + 1) / n_threads;
      for (int64_t i = lo; i < hi; ++i) body(i);
    });
  }
  for (auto& t : pool) t.join();
}

}  // namespace

extern "C" {

int oracle_hardware_threads() { return pick_threads(0); }

// Indexer scores.  q_idx [B][T][Hi][Di], w [B][T][Hi], k_idx [B][L][Di] (bf16 bits),
// q_pos [B][T].  scores [B][T][L] (double); s > q_pos gets -infinity.
// Returns 0, or -1 when a position is out of range.
int oracle_index_scores(int B, int T, int L, int Hi, int Di, const uint16_t* q_idx,
                        const uint16_t* w, const uint16_t* k_idx, const int32_t* q_pos,
                        double* scores, int n_threads) {
  for (int64_t r = 0; r < int64_t(B) * T; ++r)
    if (q_pos[r] < 0 || q_pos[r] >= L) return -1;
  const int64_t chunk = 4096;
  const int64_t chunks_per_row = (L + chunk - 1) / chunk;
  const int64_t n_items = int64_t(B) * T * chunks_per_row;
  parallel_for(n_items, pick_threads(n_threads), [&](int64_t item) {
    int64_t row = item / chunks_per_row;
    int64_t s0 = (item % chunks_per_row) * chunk;
    int64_t s1 = std::min<int64_t>(s0 + chunk, L);
    int64_t b = row / T;
    int64_t t = q_pos[row];
    std::vector<double> q(size_t(Hi) * Di), wt(Hi), k(Di);
    for (int64_t e = 0; e < int64_t(Hi) * Di; ++e) q[e] = bf16_value(q_idx[row * Hi * Di + e]);
    for (int j = 0; j < Hi; ++j) wt[j] = bf16_value(w[row * Hi + j]);
    for (int64_t s = s0; s < s1; ++s) {
      double* out = scores + row * L + s;
      if (s > t) {
        *out = -std::numeric_limits<double>::infinity();
        continue;
      }
      const uint16_t* ks = k_idx + (b * L + s) * Di;
      for (int d = 0; d < Di; ++d) k[d] = bf16_value(ks[d]);
      double total = 0.0;
      for (int j = 0; j < Hi; ++j) {
        double dot = 0.0;
        for (int d = 0; d < Di; ++d) dot += q[size_t(j) * Di + d] * k[d];
        total += wt[j] * std::max(0.0, dot);
      }
      *out = total;
    }
  });
  return 0;
}

// Top-K selection per row.  scores [rows][L] (double), q_pos [rows].
// idx [rows][K]: the selected positions in ascending order, then -1.
// Order used: larger score first, equal scores -> lower position first.
int oracle_topk(int rows, int L, const double* scores, const int32_t* q_pos, int K,
                int32_t* idx, int n_threads) {
  if (K <= 0) return -1;
  for (int r = 0; r < rows; ++r)
    if (q_pos[r] < 0 || q_pos[r] >= L) return -1;
  parallel_for(rows, pick_threads(n_threads), [&](int64_t r) {
    int64_t n = int64_t(q_pos[r]) + 1;
    int32_t* out = idx + r * int64_t(K);
    std::vector<int32_t> chosen;
    if (n <= K) {
      for (int64_t s = 0; s < n; ++s) chosen.push_back(int32_t(s));
    } else {
      const double* sc = scores + r * int64_t(L);
      std::vector<std::pair<double, int32_t>> cand(n);  // (-score, position)
      for (int64_t s = 0; s < n; ++s) cand[s] = {-sc[s], int32_t(s)};
      std::nth_element(cand.begin(), cand.begin() + (K - 1), cand.end());
      // Everything before position K-1 now orders at or before it; together
      // with it they are the K best pairs.
      for (int j = 0; j < K; ++j) chosen.push_back(cand[j].second);
      std::sort(chosen.begin(), chosen.end());
    }
    for (int j = 0; j < K; ++j) out[j] = j < int(chosen.size()) ? chosen[j] : -1;
  });
  return 0;
}

// Sparse latent attention plus the per-head sigmoid gate.
// q [B][T][H][Dq], kv [B][L][Dq], idx [B][T][K] (-1 slots skipped), gate [B][T][H]
// or null (ungated).  out [B][T][H][Dv] (double).  A query with no valid slot
// produces zeros.  Returns -1 if an index is outside [0, L).
int oracle_attend(int B, int T, int L, int H, int Dq, int Dv, double scale,
                  const uint16_t* q, const uint16_t* kv, const int32_t* idx, int K,
                  const uint16_t* gate, double* out, int n_threads) {
  for (int64_t e = 0; e < int64_t(B) * T * K; ++e)
    if (idx[e] >= L || idx[e] < -1) return -1;
  const int64_t n_items = int64_t(B) * T * H;
  parallel_for(n_items, pick_threads(n_threads), [&](int64_t item) {
    int64_t row = item / H;
    int h = int(item % H);
    int64_t b = row / T;
    const int32_t* sel = idx + row * K;
    std::vector<double> qh(Dq), c(Dq), z, acc(Dv, 0.0);
    std::vector<int32_t> pos;
    for (int d = 0; d < Dq; ++d) qh[d] = bf16_value(q[(row * H + h) * Dq + d]);
    for (int j = 0; j < K; ++j) {
      if (sel[j] < 0) continue;
      const uint16_t* cs = kv + (b * L + sel[j]) * Dq;
      double dot = 0.0;
      for (int d = 0; d < Dq; ++d) dot += qh[d] * bf16_value(cs[d]);
      z.push_back(dot * scale);
      pos.push_back(sel[j]);
    }
    double* o = out + (row * H + h) * Dv;
    if (z.empty()) {
      for (int d = 0; d < Dv; ++d) o[d] = 0.0;
      return;
    }
    double m = *std::max_element(z.begin(), z.end());
    double denom = 0.0;
    for (size_t j = 0; j < z.size(); ++j) {
      double p = std::exp(z[j] - m);
      denom += p;
      const uint16_t* cs = kv + (b * L + pos[j]) * Dq;
      for (int d = 0; d < Dv; ++d) acc[d] += p * bf16_value(cs[d]);
    }
    double g = 1.0;
    if (gate) g = 1.0 / (1.0 + std::exp(-bf16_value(gate[row * H + h])));
    for (int d = 0; d < Dv; ++d) o[d] = acc[d] / denom * g;
  });
  return 0;
}

// The whole path: indexer -> top-K -> attention with gate.  scores_out and
// idx_out may be null; when given they receive the intermediate results.
int oracle_forward(int B, int T, int L, int Hi, int Di, int H, int Dq, int Dv, double scale,
                   int K, const uint16_t* q_idx, const uint16_t* w, const uint16_t* k_idx,
                   const uint16_t* q, const uint16_t* kv, const uint16_t* gate,
                   const int32_t* q_pos, int32_t* idx_out, double* out, int n_threads) {
  std::vector<double> scores(size_t(B) * T * L);
  std::vector<int32_t> idx(size_t(B) * T * K);
  int rc = oracle_index_scores(B, T, L, Hi, Di, q_idx, w, k_idx, q_pos, scores.data(), n_threads);
  if (rc) return rc;
  rc = oracle_topk(B * T, L, scores.data(), q_pos, K, idx.data(), n_threads);
  if (rc) return rc;
  if (idx_out) std::memcpy(idx_out, idx.data(), idx.size() * sizeof(int32_t));
  return oracle_attend(B, T, L, H, Dq, Dv, scale, q, kv, idx.data(), K, gate, out, n_threads);
}

}  // extern "C"
