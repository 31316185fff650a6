// Launch interfaces between the C-ABI layer (sga_api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sga.h"

namespace sga {

// sga_forward that also writes the attention output rounded to bf16 (nearest
// even) into out_bf16 [rows][64][512] (8-byte aligned): the whole layer's W_UV
// input, without a conversion pass.  Arguments otherwise as sga_forward's.
sga_status_t forward_bf16_copy(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                               const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                               const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out,
                               uint16_t* out_bf16, void* ws, size_t ws_bytes, sga_stream_t stream);

// ---- indexer (step 1) --------------------------------------------------------
struct IndexArgs {
  const void* q_idx;      // [rows][64][128] bf16, or E4M3 bytes when fp8
  const uint16_t* w;      // [rows][64]
  const void* k_idx;      // [B][L][128] bf16, or E4M3 bytes when fp8
  const int32_t* q_pos;   // [rows]
  float* scores;          // [rows][L]; not written when `cand` is set
  uint32_t* hist;         // [rows][4096] first-level top-k histogram (all zero on entry) or null
  int* status;
  int batch, n_q, kv_stride;
  bool fp8;               // indexer queries and keys in E4M3
  // Selection candidates instead of scores (decode only, with `hist`; see
  // fused_topk_ok): row r appends (order key << 32 | position) to
  // cand[r][0 .. L) for every key that can still be among its top_k, counting
  // them in cand_n[r * kCandNStride] (zero on entry).  `hist` then counts only
  // those keys: exact for every bin at or above the K-th key's bin.
  uint64_t* cand = nullptr;
  uint32_t* cand_n = nullptr;
  int top_k = 0;
};
// n_q >= 8 queries per sequence take the prefill kernel (query blocks x key
// tiles), which counts no histogram: `hist` is then ignored.
cudaError_t launch_index_scores(const IndexArgs& a, int num_sms, cudaStream_t stream);
bool index_uses_prefill(int n_q);
// The fused selection (the indexer emits candidates, a per-row kernel selects
// from them) takes decode rows of at most kFusedTopkMaxL positions.
constexpr int kFusedTopkMaxL = 262144;
// Candidate counters are kCandNStride words apart: one 128-byte line per row,
// so the rows' counter updates spread over L2 slices.
constexpr int kCandNStride = 32;
inline bool fused_topk_ok(int n_q, int kv_stride) { return !index_uses_prefill(n_q) && kv_stride <= kFusedTopkMaxL; }

// ---- top-k (step 2) ------------------------------------------------------------
struct TopkArgs {
  const float* scores;   // [rows][L]
  const int32_t* q_pos;  // [rows]
  int32_t* idx;          // [rows][K]
  uint32_t* bitmap;      // [rows][words_per_row] scratch
  uint32_t* hist;        // [rows][4096] histogram of the top 12 order bits, or null; zeroed after use
  int* status;
  int rows, kv_stride, top_k;
};
size_t topk_bitmap_words(int kv_stride);
int topk_cluster_size(int rows);
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream);

// The selection from the indexer's candidates (rows of at most kFusedTopkMaxL
// positions): one CTA per row; clears hist[r] and cand_n[r] for the next call.
struct TopkCandArgs {
  const uint64_t* cand;  // [rows][L]: (order key << 32 | position), cand_n[r] of them
  uint32_t* cand_n;      // [rows][kCandNStride], word 0 of each row
  uint32_t* hist;        // [rows][4096] first-level histograms, exact at and above the K-th key's bin
  const int32_t* q_pos;  // [rows]
  int32_t* idx;          // [rows][K]
  int* status;
  int rows, kv_stride, top_k;
};
cudaError_t launch_topk_candidates(const TopkCandArgs& a, cudaStream_t stream);

// ---- sparse attention + gate (steps 3-4) -----------------------------------------
struct AttendArgs {
  const uint16_t* q;     // [rows][64][576]
  const uint16_t* kv;    // [B][L][576]
  const int32_t* idx;    // [rows][K]
  const uint16_t* gate;  // [rows][64] or null
  float* out;            // [rows][64][512]
  int* status;
  int batch, n_q, kv_stride, top_k;
  uint16_t* out_bf16 = nullptr;  // [rows][64][512]: out rounded to bf16 (nearest even) as well, or null
};
int attend_splits(int rows, int top_k);
cudaError_t launch_attend(const AttendArgs& a, cudaStream_t stream);

// ---- the layer's projections: weight-streaming GEMM -----------------------------------
// Y[b][n][m] = sum_k X[n][x_col_per_batch * b + k] W[b](m, k), W row-major
// [batch][m][k] (K-major) or [batch][k][m] (MN-major), bf16 in, fp32 accumulate.
constexpr int kGemmMaxN = 128;  // tokens per work item (more tokens: several items)
struct GemmArgs {
  const uint16_t* w;
  const uint16_t* x;     // [n][x_ld] bf16 (x_ld * 2 bytes a multiple of 16)
  int m, n, k, batch;
  bool w_mn_major;
  int x_ld, x_col_per_batch;
  int splits;            // K splits: fp32 partials, added by the consumer in split order
  float* part;           // fp32 output part[split][n][batch * m], or null
  uint16_t* out;         // bf16 output out[col * out_ld + b * out_boff + m] (splits == 1), or null
  int out_ld, out_boff;
  int* status;
};
// K splits that keep `num_sms` SMs streaming when there are fewer tiles than SMs.
int gemm_splits(int m, int n, int k, int batch, int num_sms);
cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream);

// ---- tensor maps -------------------------------------------------------------------
// 2-D bf16 tensor map: `inner` elements per row, `outer` rows, rows `row_bytes`
// apart, box {box_inner, box_outer}, 128-byte swizzle.
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
// Same, over bytes (E4M3 values) when `bytes`, else bf16.
cudaError_t make_tmap_2d(CUtensorMap* map, bool bytes, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

}  // namespace sga
