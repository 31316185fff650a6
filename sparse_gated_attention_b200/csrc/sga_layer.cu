// The projections either side of the hot path: one SGA attention layer over
// new tokens (archdb "A.X K2", attention fields: 64 heads, qk head dim 192 =
// 128 nope + 64 rope, v head dim 128, KV latent 512, q low-rank width 1536,
// a 64-dim decoupled RoPE key shared across heads, RoPE base 1e6, no QK norm,
// no projection bias; gate field: a head-specific sigmoid gate before o_proj,
// projected jointly with the query; token-selection field: a DSA-style indexer
// with 64 heads of dim 128).
//
//   G1  [c_q | c_kv, k_rope | k_idx | w] = W_hq h            (one GEMM, m = R + 768)
//   P1  bf16 rounding; RoPE on k_rope; the cache rows written at each token's
//       position; c_q and w kept for the next steps
//   G2  [q_nope, q_rope per head | g | q_idx] = W_cq c_q      (one GEMM, m = 20,544)
//   P2  bf16 rounding; RoPE on q_rope (into q's last 64 dims); gate, q_idx
//   G3  q_lat[h] = W_UK[h]^T q_nope[h]                        (64 batched GEMMs)
//   C   q_lat -> q's first 512 dims (bf16)
//   path: sga_forward (indexer, top-2048, latent attention + gate)
//   C   out -> bf16
//   G4  o[h] = W_UV[h] out[h]                                  (64 batched GEMMs)
//   C   o -> bf16
//   G5  y = W_O o                                             (m = d_model)
//
// Every activation between two contractions is rounded to bf16 (round to
// nearest even), the precision of the cached rows; the GEMMs accumulate in
// fp32.  The GEMMs are plain library GEMMs (cuBLAS, bf16 inputs, fp32
// output); the packing, rounding and rotation steps are the kernels below.
//
// RoPE: interleaved pairs (2i, 2i+1), i < 32, rotated by p * 1e6^(-i/32) at
// the token's absolute position p.  The angle is formed and reduced in double
// precision (p reaches 2^18, so an fp32 angle would be off by ~1e-2 rad), the
// rotation itself runs in fp32 on the bf16-rounded inputs.
#include <cublas_v2.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "../../include/sga.h"
#include "sga_host.h"

namespace {

constexpr int kHeads = SGA_HEADS;          // 64
constexpr int kNope = 128;
constexpr int kRope = 64;
constexpr int kLatent = SGA_V_DIM;         // 512
constexpr int kKvDim = SGA_QK_DIM;         // 576
constexpr int kVHead = 128;
constexpr int kIdxHeads = SGA_INDEX_HEADS;  // 64
constexpr int kIdxDim = SGA_INDEX_DIM;      // 128
constexpr int kQRows = kHeads * (kNope + kRope);                  // 12,288
constexpr int kCqRows = kQRows + kHeads + kIdxHeads * kIdxDim;    // 20,544
constexpr int kHqExtra = kKvDim + kIdxDim + kIdxHeads;            // 768
constexpr int kOWidth = kHeads * kVHead;                          // 8,192
constexpr double kRopeBase = 1.0e6;

using sga::host::align_up;
using sga::host::aligned;
using sga::host::at;
using sga::host::kStatusBytes;
constexpr size_t kAlign = sga::host::kWsAlign;
constexpr size_t kCublasWs = 32u << 20;


__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// cos and sin of pos * base^(-i/32), formed in double precision.
__device__ __forceinline__ void rope_angle(int pos, int i, float* c, float* s) {
  const double theta = pow(kRopeBase, -static_cast<double>(i) / (kRope / 2));
  double sd, cd;
  sincos(static_cast<double>(pos) * theta, &sd, &cd);
  *c = static_cast<float>(cd);
  *s = static_cast<float>(sd);
}

// Rotates the bf16-rounded pair (x, y) and returns the two bf16 results.
__device__ __forceinline__ void rope_pair(float x, float y, int pos, int i, uint16_t* o0, uint16_t* o1) {
  float c, s;
  rope_angle(pos, i, &c, &s);
  x = round_bf16(x);
  y = round_bf16(y);
  *o0 = bf16_bits(x * c - y * s);
  *o1 = bf16_bits(x * s + y * c);
}

struct PrepHArgs {
  const float* g1;       // [rows][R + 768]
  const int32_t* q_pos;  // [rows]
  uint16_t* c_q;         // [rows][R]
  uint16_t* kv_cache;    // [B][L][576]
  uint16_t* kidx_cache;  // [B][L][128]
  uint16_t* w;           // [rows][64]
  int* status;
  int R, n_q, L;
};

// One block per new token: c_q, w, and its cache rows (c_kv, rotated k_rope, k_idx).
__global__ void layer_prep_h_kernel(PrepHArgs a) {
  const int row = blockIdx.x;
  const int b = row / a.n_q;
  const int pos = a.q_pos[row];
  const int ld = a.R + kHqExtra;
  const float* g = a.g1 + static_cast<size_t>(row) * ld;
  for (int j = threadIdx.x; j < a.R; j += blockDim.x) a.c_q[static_cast<size_t>(row) * a.R + j] = bf16_bits(g[j]);
  for (int j = threadIdx.x; j < kIdxHeads; j += blockDim.x)
    a.w[static_cast<size_t>(row) * kIdxHeads + j] = bf16_bits(g[a.R + kKvDim + kIdxDim + j]);
  if (pos < 0 || pos >= a.L) {
    if (threadIdx.x == 0) atomicCAS(a.status, 0, SGA_ERR_DEVICE_ARG);
    return;
  }
  const size_t cache_row = static_cast<size_t>(b) * a.L + pos;
  uint16_t* kv = a.kv_cache + cache_row * kKvDim;
  for (int j = threadIdx.x; j < kLatent; j += blockDim.x) kv[j] = bf16_bits(g[a.R + j]);
  for (int i = threadIdx.x; i < kRope / 2; i += blockDim.x)
    rope_pair(g[a.R + kLatent + 2 * i], g[a.R + kLatent + 2 * i + 1], pos, i, &kv[kLatent + 2 * i],
              &kv[kLatent + 2 * i + 1]);
  uint16_t* ki = a.kidx_cache + cache_row * kIdxDim;
  for (int j = threadIdx.x; j < kIdxDim; j += blockDim.x) ki[j] = bf16_bits(g[a.R + kKvDim + j]);
}

struct PrepQArgs {
  const float* g2;       // [rows][20544]
  const int32_t* q_pos;  // [rows]
  uint16_t* q_nope;      // [rows][64][128]
  uint16_t* q;           // [rows][64][576]: rotated q_rope into dims 512..575
  uint16_t* gate;        // [rows][64]
  uint16_t* q_idx;       // [rows][64][128]
};

// One block per new token: q_nope, the rotated q_rope, the gate logits and the indexer query.
__global__ void layer_prep_q_kernel(PrepQArgs a) {
  const int row = blockIdx.x;
  const int pos = a.q_pos[row];  // range-checked where the caches are written; only the angle uses it here
  const float* g = a.g2 + static_cast<size_t>(row) * kCqRows;
  for (int j = threadIdx.x; j < kHeads * kNope; j += blockDim.x) {
    const int h = j / kNope, d = j - h * kNope;
    a.q_nope[static_cast<size_t>(row) * kHeads * kNope + j] = bf16_bits(g[h * (kNope + kRope) + d]);
  }
  for (int j = threadIdx.x; j < kHeads * (kRope / 2); j += blockDim.x) {
    const int h = j / (kRope / 2), i = j - h * (kRope / 2);
    const float* src = g + h * (kNope + kRope) + kNope + 2 * i;
    uint16_t* dst = a.q + (static_cast<size_t>(row) * kHeads + h) * kKvDim + kLatent + 2 * i;
    rope_pair(src[0], src[1], pos, i, &dst[0], &dst[1]);
  }
  for (int j = threadIdx.x; j < kHeads; j += blockDim.x)
    a.gate[static_cast<size_t>(row) * kHeads + j] = bf16_bits(g[kQRows + j]);
  for (int j = threadIdx.x; j < kIdxHeads * kIdxDim; j += blockDim.x)
    a.q_idx[static_cast<size_t>(row) * kIdxHeads * kIdxDim + j] = bf16_bits(g[kQRows + kHeads + j]);
}

// dst[r][c] = bf16(src[r][c]) for r < n_rows, c < n_cols (n_cols a multiple of 4, strides of 4 elements).
__global__ void f32_to_bf16_rows_kernel(const float* src, int src_ld, uint16_t* dst, int dst_ld, int n_rows,
                                        int n_cols) {
  const int vec_per_row = n_cols / 4;
  const long long total = static_cast<long long>(n_rows) * vec_per_row;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(e / vec_per_row), c = static_cast<int>(e - static_cast<long long>(r) * vec_per_row);
    const float4 v = *reinterpret_cast<const float4*>(src + static_cast<size_t>(r) * src_ld + 4 * c);
    const uint32_t lo = bf16_bits(v.x) | (static_cast<uint32_t>(bf16_bits(v.y)) << 16);
    const uint32_t hi = bf16_bits(v.z) | (static_cast<uint32_t>(bf16_bits(v.w)) << 16);
    *reinterpret_cast<uint2*>(dst + static_cast<size_t>(r) * dst_ld + 4 * c) = make_uint2(lo, hi);
  }
}

cudaError_t launch_convert(const float* src, int src_ld, uint16_t* dst, int dst_ld, int n_rows, int n_cols,
                           cudaStream_t s) {
  const long long total = static_cast<long long>(n_rows) * (n_cols / 4);
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 8));
  f32_to_bf16_rows_kernel<<<blocks, 256, 0, s>>>(src, src_ld, dst, dst_ld, n_rows, n_cols);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- cuBLAS
// One handle per device, created on first use (outside stream capture) and
// kept for the life of the process; every call sets its stream and points its
// workspace into the caller's workspace, so cuBLAS allocates nothing itself.
std::mutex g_cublas_mu;
cublasHandle_t g_cublas[64] = {};

cublasHandle_t cublas_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(g_cublas_mu);
  if (!g_cublas[dev]) {
    cublasHandle_t h = nullptr;
    if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
    g_cublas[dev] = h;
  }
  return g_cublas[dev];
}

// Row-major Y[n][m] = X[n][k] W[m][k]^T (column-major: Y^T = W X^T with W read transposed).
cublasStatus_t gemm_xwt(cublasHandle_t h, int m, int n, int k, const uint16_t* W, const uint16_t* X, float* Y) {
  const float one = 1.f, zero = 0.f;
  return cublasGemmEx(h, CUBLAS_OP_T, CUBLAS_OP_N, m, n, k, &one, W, CUDA_R_16BF, k, X, CUDA_R_16BF, k, &zero, Y,
                      CUDA_R_32F, m, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT);
}

// ---------------------------------------------------------------- workspace
struct LayerLayout {
  size_t path = 0;  // sga_forward's workspace (its status word is the layer's)
  size_t cublas = 0, g1 = 0, c_q = 0, g2 = 0, q_nope = 0, q_lat = 0, q = 0, gate = 0, q_idx = 0, w = 0;
  size_t out = 0, out_b = 0, o = 0, o_b = 0, total = 0;
};

bool layer_dims_ok(const sga_dims_t* d, const sga_layer_weights_t* W) {
  if (!d || !W) return false;
  if (d->batch < 1 || d->n_q < 1 || d->kv_stride < 1 || d->kv_stride > SGA_MAX_KV_STRIDE) return false;
  if (W->d_model < 8 || W->d_model % 8 != 0 || W->q_rank < 8 || W->q_rank % 8 != 0) return false;
  const long long rows = static_cast<long long>(d->batch) * d->n_q;
  if (rows * kCqRows > INT32_MAX || rows * kHeads * kLatent > INT32_MAX) return false;
  if (static_cast<long long>(d->batch) * d->kv_stride > INT32_MAX) return false;
  return true;
}

// op: SGA_LAYER_PROJECT, SGA_LAYER_OUTPUT or SGA_LAYER_FORWARD (covers both).
sga_status_t layer_layout(const sga_dims_t& d, int q_rank, sga_layer_op_t op, LayerLayout* l) {
  const size_t rows = static_cast<size_t>(d.batch) * d.n_q;
  size_t off = kStatusBytes;
  if (op == SGA_LAYER_FORWARD) {
    size_t path_bytes = 0;
    if (d.top_k < 64 || d.top_k > SGA_MAX_TOP_K || d.top_k % 64 != 0) return SGA_ERR_INVALID_ARG;
    const sga_status_t st = sga_workspace_size(&d, SGA_OP_FORWARD, &path_bytes);
    if (st != SGA_OK) return st;
    l->path = 0;
    off = align_up(path_bytes);
  }
  l->cublas = off;
  off += kCublasWs;
  if (op != SGA_LAYER_OUTPUT) {
    l->g1 = off;
    off += align_up(rows * (q_rank + kHqExtra) * 4);
    l->c_q = off;
    off += align_up(rows * q_rank * 2);
    l->g2 = off;
    off += align_up(rows * kCqRows * 4);
    l->q_nope = off;
    off += align_up(rows * kHeads * kNope * 2);
    l->q_lat = off;
    off += align_up(rows * kHeads * kLatent * 4);
  }
  if (op == SGA_LAYER_FORWARD) {
    l->q = off;
    off += align_up(rows * kHeads * kKvDim * 2);
    l->gate = off;
    off += align_up(rows * kHeads * 2);
    l->q_idx = off;
    off += align_up(rows * kIdxHeads * kIdxDim * 2);
    l->w = off;
    off += align_up(rows * kIdxHeads * 2);
    l->out = off;
    off += align_up(rows * kHeads * kLatent * 4);
  }
  if (op != SGA_LAYER_PROJECT) {
    l->out_b = off;
    off += align_up(rows * kHeads * kLatent * 2);
    l->o = off;
    off += align_up(rows * kOWidth * 4);
    l->o_b = off;
    off += align_up(rows * kOWidth * 2);
  }
  l->total = off;
  return SGA_OK;
}

bool weights_ok(const sga_layer_weights_t* W, bool front, bool back) {
  if (front && (!aligned(W->w_hq, 16) || !aligned(W->w_cq, 16) || !aligned(W->w_uk, 16))) return false;
  if (back && (!aligned(W->w_uv, 16) || !aligned(W->w_o, 16))) return false;
  return true;
}

sga_status_t device_ok() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
                                                cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  return major == 10 ? SGA_OK : SGA_ERR_UNSUPPORTED;
}

sga_status_t begin(void* ws, const LayerLayout& l, cudaStream_t s, cublasHandle_t* h) {
  *h = cublas_for_current_device();
  if (!*h) return SGA_ERR_CUDA;
  if (cublasSetStream(*h, s) != CUBLAS_STATUS_SUCCESS) return SGA_ERR_CUDA;
  if (cublasSetWorkspace(*h, at<void>(ws, l.cublas), kCublasWs) != CUBLAS_STATUS_SUCCESS) return SGA_ERR_CUDA;
  return SGA_OK;
}

// G1, P1, G2, P2, G3 and the q_lat conversion: the path's inputs for the new tokens.
sga_status_t project_impl(const sga_dims_t& d, const sga_layer_weights_t* W, const uint16_t* h, const int32_t* q_pos,
                          uint16_t* kv_cache, uint16_t* kidx_cache, uint16_t* q, uint16_t* gate, uint16_t* q_idx,
                          uint16_t* w, void* ws, const LayerLayout& l, cublasHandle_t hb, cudaStream_t s) {
  const int rows = d.batch * d.n_q;
  const int R = W->q_rank;
  float* g1 = at<float>(ws, l.g1);
  uint16_t* c_q = at<uint16_t>(ws, l.c_q);
  float* g2 = at<float>(ws, l.g2);
  uint16_t* q_nope = at<uint16_t>(ws, l.q_nope);
  float* q_lat = at<float>(ws, l.q_lat);
  if (gemm_xwt(hb, R + kHqExtra, rows, W->d_model, W->w_hq, h, g1) != CUBLAS_STATUS_SUCCESS) return SGA_ERR_CUDA;
  PrepHArgs pa{g1, q_pos, c_q, kv_cache, kidx_cache, w, at<int>(ws, 0), R, d.n_q, d.kv_stride};
  layer_prep_h_kernel<<<rows, 256, 0, s>>>(pa);
  if (cudaGetLastError() != cudaSuccess) return SGA_ERR_CUDA;
  if (gemm_xwt(hb, kCqRows, rows, R, W->w_cq, c_q, g2) != CUBLAS_STATUS_SUCCESS) return SGA_ERR_CUDA;
  PrepQArgs qa{g2, q_pos, q_nope, q, gate, q_idx};
  layer_prep_q_kernel<<<rows, 256, 0, s>>>(qa);
  if (cudaGetLastError() != cudaSuccess) return SGA_ERR_CUDA;
  // q_lat[r][h][j] = sum_d W_UK[h][d][j] q_nope[r][h][d], per head h (column-major: C = A B,
  // A = W_UK[h] viewed as [512 x 128] with ld 512, B = q_nope[:, h, :] as [128 x rows] with ld 8192)
  const float one = 1.f, zero = 0.f;
  if (cublasGemmStridedBatchedEx(hb, CUBLAS_OP_N, CUBLAS_OP_N, kLatent, rows, kNope, &one, W->w_uk, CUDA_R_16BF,
                                 kLatent, static_cast<long long>(kNope) * kLatent, q_nope, CUDA_R_16BF, kHeads * kNope,
                                 kNope, &zero, q_lat, CUDA_R_32F, kHeads * kLatent, kLatent, kHeads,
                                 CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return SGA_ERR_CUDA;
  return launch_convert(q_lat, kLatent, q, kKvDim, rows * kHeads, kLatent, s) == cudaSuccess ? SGA_OK : SGA_ERR_CUDA;
}

// out -> bf16, G4 (W_UV per head), o -> bf16, G5 (o_proj).
sga_status_t output_impl(const sga_dims_t& d, const sga_layer_weights_t* W, const float* out, float* y, void* ws,
                         const LayerLayout& l, cublasHandle_t hb, cudaStream_t s) {
  const int rows = d.batch * d.n_q;
  uint16_t* out_b = at<uint16_t>(ws, l.out_b);
  float* o = at<float>(ws, l.o);
  uint16_t* o_b = at<uint16_t>(ws, l.o_b);
  if (launch_convert(out, kLatent, out_b, kLatent, rows * kHeads, kLatent, s) != cudaSuccess) return SGA_ERR_CUDA;
  // o[r][h][i] = sum_j W_UV[h][i][j] out[r][h][j] (column-major: A = W_UV[h] stored [512 x 128], read
  // transposed; B = out[:, h, :] as [512 x rows] with ld 32768; C = o[:, h, :] as [128 x rows] with ld 8192)
  const float one = 1.f, zero = 0.f;
  if (cublasGemmStridedBatchedEx(hb, CUBLAS_OP_T, CUBLAS_OP_N, kVHead, rows, kLatent, &one, W->w_uv, CUDA_R_16BF,
                                 kLatent, static_cast<long long>(kVHead) * kLatent, out_b, CUDA_R_16BF,
                                 kHeads * kLatent, kLatent, &zero, o, CUDA_R_32F, kOWidth, kVHead, kHeads,
                                 CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS)
    return SGA_ERR_CUDA;
  if (launch_convert(o, kOWidth, o_b, kOWidth, rows, kOWidth, s) != cudaSuccess) return SGA_ERR_CUDA;
  return gemm_xwt(hb, W->d_model, rows, kOWidth, W->w_o, o_b, y) == CUBLAS_STATUS_SUCCESS ? SGA_OK : SGA_ERR_CUDA;
}

sga_status_t check_layer_ws(void* ws, size_t ws_bytes, const sga_dims_t& d, int q_rank, sga_layer_op_t op,
                            LayerLayout* l) {
  const sga_status_t st = layer_layout(d, q_rank, op, l);
  if (st != SGA_OK) return st;
  if (!aligned(ws, kAlign) || ws_bytes < l->total) return SGA_ERR_WORKSPACE;
  return SGA_OK;
}

}  // namespace

extern "C" {

sga_status_t sga_layer_workspace_size(const sga_dims_t* dims, const sga_layer_weights_t* weights, sga_layer_op_t op,
                                      size_t* bytes) {
  if (!bytes || !layer_dims_ok(dims, weights)) return SGA_ERR_INVALID_ARG;
  if (op != SGA_LAYER_PROJECT && op != SGA_LAYER_OUTPUT && op != SGA_LAYER_FORWARD) return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  const sga_status_t st = layer_layout(*dims, weights->q_rank, op, &l);
  if (st != SGA_OK) return st;
  *bytes = l.total;
  return SGA_OK;
}

sga_status_t sga_layer_project(const sga_dims_t* dims, const sga_layer_weights_t* weights, const sga_bf16_t* h,
                               const int32_t* q_pos, sga_bf16_t* kv_cache, sga_bf16_t* k_idx_cache, sga_bf16_t* q,
                               sga_bf16_t* gate, sga_bf16_t* q_idx, sga_bf16_t* w, void* ws, size_t ws_bytes,
                               sga_stream_t stream) {
  if (!layer_dims_ok(dims, weights) || !weights_ok(weights, true, false)) return SGA_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(q_pos, 4) || !aligned(kv_cache, 16) || !aligned(k_idx_cache, 16) ||
      !aligned(q, 16) || !aligned(gate, 16) || !aligned(q_idx, 16) || !aligned(w, 16))
    return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights->q_rank, SGA_LAYER_PROJECT, &l);
  if (st != SGA_OK) return st;
  if ((st = device_ok()) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle_t hb;
  if ((st = begin(ws, l, s, &hb)) != SGA_OK) return st;
  return project_impl(*dims, weights, h, q_pos, kv_cache, k_idx_cache, q, gate, q_idx, w, ws, l, hb, s);
}

sga_status_t sga_layer_output(const sga_dims_t* dims, const sga_layer_weights_t* weights, const float* out, float* y,
                              void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!layer_dims_ok(dims, weights) || !weights_ok(weights, false, true)) return SGA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(y, 16)) return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights->q_rank, SGA_LAYER_OUTPUT, &l);
  if (st != SGA_OK) return st;
  if ((st = device_ok()) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle_t hb;
  if ((st = begin(ws, l, s, &hb)) != SGA_OK) return st;
  return output_impl(*dims, weights, out, y, ws, l, hb, s);
}

sga_status_t sga_layer_forward(const sga_dims_t* dims, const sga_layer_weights_t* weights, const sga_bf16_t* h,
                               const int32_t* q_pos, sga_bf16_t* kv_cache, sga_bf16_t* k_idx_cache, int32_t* idx_out,
                               float* y, void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!layer_dims_ok(dims, weights) || !weights_ok(weights, true, true)) return SGA_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(q_pos, 4) || !aligned(kv_cache, 16) || !aligned(k_idx_cache, 16) ||
      !aligned(y, 16) || (idx_out && !aligned(idx_out, 16)))
    return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights->q_rank, SGA_LAYER_FORWARD, &l);
  if (st != SGA_OK) return st;
  if ((st = device_ok()) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cublasHandle_t hb;
  if ((st = begin(ws, l, s, &hb)) != SGA_OK) return st;
  uint16_t* q = at<uint16_t>(ws, l.q);
  uint16_t* gate = at<uint16_t>(ws, l.gate);
  uint16_t* q_idx = at<uint16_t>(ws, l.q_idx);
  uint16_t* w = at<uint16_t>(ws, l.w);
  float* out = at<float>(ws, l.out);
  st = project_impl(*dims, weights, h, q_pos, kv_cache, k_idx_cache, q, gate, q_idx, w, ws, l, hb, s);
  if (st != SGA_OK) return st;
  size_t path_bytes = 0;
  sga_workspace_size(dims, SGA_OP_FORWARD, &path_bytes);
  st = sga_forward(dims, q_idx, w, k_idx_cache, q, kv_cache, gate, q_pos, idx_out, out, ws, path_bytes, stream);
  if (st != SGA_OK) return st;
  return output_impl(*dims, weights, out, y, ws, l, hb, s);
}

}  // extern "C"
