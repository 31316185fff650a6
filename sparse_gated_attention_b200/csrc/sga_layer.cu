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
//   G3  q_lat[h] = W_UK[h]^T q_nope[h], rounded to bf16 into q's first 512 dims
//       (64 heads, MN-major weights)
//   path: sga_forward (indexer, top-2048, latent attention + gate)
//   C   out -> bf16
//   G4  o[h] = W_UV[h] out[h], rounded to bf16                  (64 heads)
//   G5  y = W_O o                                             (m = d_model)
//
// Every activation between two contractions is rounded to bf16 (round to
// nearest even), the precision of the cached rows; the GEMMs accumulate in
// fp32.  Every GEMM is the weight-streaming tcgen05 kernel of sga_gemm.cu: the
// weights (230 MB at the model's widths) are streamed once through TMA while
// the new tokens sit in the N dimension.  G1, G2 and G5 split K when they have
// fewer 128-row tiles than SMs; their fp32 partial sums are added in split
// order by the kernels that consume them (P1, P2, the y sum), so results do
// not depend on scheduling.  G3 and G4 write bf16 straight into the layout the
// next step reads.
//
// RoPE: interleaved pairs (2i, 2i+1), i < 32, rotated by p * 1e6^(-i/32) at
// the token's absolute position p.  The angle is formed and reduced in double
// precision (p reaches 2^18, so an fp32 angle would be off by ~1e-2 rad), the
// rotation itself runs in fp32 on the bf16-rounded inputs.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>

#include "../../include/sga.h"
#include "sga_host.h"
#include "sga_internal.cuh"

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
// The K splits (and so the workspace) are chosen for a 148-SM B200 whatever the
// device; the kernels themselves run on any number of SMs.
constexpr int kSplitSms = 148;


// Programmatic dependent launch: every kernel of the layer waits here for the
// previous kernel's results, then lets the next kernel be scheduled (it waits
// in turn), so a GEMM's first weight loads overlap the kernel before it.
__device__ __forceinline__ void grid_dependency_wait_layer() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }
__device__ __forceinline__ uint16_t bf16_bits(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }

// The RoPE frequencies base^(-i/32), i < 32, computed once on the host in double precision.
struct RopeFreqs {
  double f[kRope / 2];
};

RopeFreqs rope_freqs() {
  RopeFreqs r;
  for (int i = 0; i < kRope / 2; ++i) r.f[i] = std::pow(kRopeBase, -static_cast<double>(i) / (kRope / 2));
  return r;
}

// cos and sin of pos * freq, formed and reduced in double precision (pos reaches
// 2^18, so an fp32 angle would be off by ~1e-2 rad).
__device__ __forceinline__ void rope_cs(int pos, double freq, float* c, float* s) {
  double sd, cd;
  sincos(static_cast<double>(pos) * freq, &sd, &cd);
  *c = static_cast<float>(cd);
  *s = static_cast<float>(sd);
}

// Rotates the bf16-rounded pair (x, y) by (c, s) and returns the two bf16 results.
__device__ __forceinline__ void rope_rotate(float x, float y, float c, float s, uint16_t* o0, uint16_t* o1) {
  x = round_bf16(x);
  y = round_bf16(y);
  *o0 = bf16_bits(x * c - y * s);
  *o1 = bf16_bits(x * s + y * c);
}

struct PrepHArgs {
  const float* g1;       // [splits][rows][R + 768] partial sums
  const int32_t* q_pos;  // [rows]
  uint16_t* c_q;         // [rows][R]
  uint16_t* kv_cache;    // [B][L][576]
  uint16_t* kidx_cache;  // [B][L][128]
  uint16_t* w;           // [rows][64]
  int* status;
  int R, n_q, L, splits;
  size_t split_stride;   // elements between consecutive partial-sum arrays
  RopeFreqs freqs;
};

// The sum of a GEMM output's `splits` partials, in split order.
// Split partials of one GEMM output element (at most kMaxGemmSplits of them,
// the bound gemm_splits keeps): all loads issued before the first add, then
// added in split order.
constexpr int kMaxGemmSplits = 8;
struct Partials {
  const float* base;
  int splits;
  size_t stride;
  __device__ __forceinline__ float operator[](size_t i) const {
    float u[kMaxGemmSplits];
#pragma unroll
    for (int s = 0; s < kMaxGemmSplits; ++s) u[s] = s < splits ? base[static_cast<size_t>(s) * stride + i] : 0.f;
    float v = u[0];
#pragma unroll
    for (int s = 1; s < kMaxGemmSplits; ++s)
      if (s < splits) v += u[s];
    return v;
  }
};

// Blocks per token: enough threads that each takes one or two items, so the
// summed split partials of an item are the only memory round trips in its chain.
constexpr int kPrepHParts = 9;   // 2,272 items per token with R = 1536
constexpr int kPrepQParts = 36;  // 18,496 items per token

// Blocks (token, part): c_q, w and the token's cache rows (c_kv, rotated
// k_rope, k_idx), the elements of a token dealt round-robin over its parts.
__global__ void layer_prep_h_kernel(PrepHArgs a) {
  grid_dependency_wait_layer();
  const int row = blockIdx.x;
  const int b = row / a.n_q;
  const int pos = a.q_pos[row];
  const int ld = a.R + kHqExtra;
  const Partials g{a.g1 + static_cast<size_t>(row) * ld, a.splits, a.split_stride};
  const bool cache = pos >= 0 && pos < a.L;
  if (!cache && threadIdx.x == 0 && blockIdx.y == 0) atomicCAS(a.status, 0, SGA_ERR_DEVICE_ARG);
  const size_t cache_row = static_cast<size_t>(b) * a.L + (cache ? pos : 0);
  uint16_t* kv = a.kv_cache + cache_row * kKvDim;
  uint16_t* ki = a.kidx_cache + cache_row * kIdxDim;
  // items: c_q (R) | w (64) | c_kv (512) | k_idx (128) | rope pairs (32)
  const int n_items = a.R + kIdxHeads + (cache ? kLatent + kIdxDim + kRope / 2 : 0);
  for (int e = blockIdx.y * blockDim.x + threadIdx.x; e < n_items; e += kPrepHParts * blockDim.x) {
    int j = e;
    if (j < a.R) {
      a.c_q[static_cast<size_t>(row) * a.R + j] = bf16_bits(g[j]);
      continue;
    }
    j -= a.R;
    if (j < kIdxHeads) {
      a.w[static_cast<size_t>(row) * kIdxHeads + j] = bf16_bits(g[a.R + kKvDim + kIdxDim + j]);
      continue;
    }
    j -= kIdxHeads;
    if (j < kLatent) {
      kv[j] = bf16_bits(g[a.R + j]);
      continue;
    }
    j -= kLatent;
    if (j < kIdxDim) {
      ki[j] = bf16_bits(g[a.R + kKvDim + j]);
      continue;
    }
    j -= kIdxDim;  // rope pair j
    float c, sn;
    rope_cs(pos, a.freqs.f[j], &c, &sn);
    rope_rotate(g[a.R + kLatent + 2 * j], g[a.R + kLatent + 2 * j + 1], c, sn, &kv[kLatent + 2 * j],
                &kv[kLatent + 2 * j + 1]);
  }
}

struct PrepQArgs {
  const float* g2;       // [splits][rows][20544] partial sums
  const int32_t* q_pos;  // [rows]
  uint16_t* q_nope;      // [rows][64][128]
  uint16_t* q;           // [rows][64][576]: rotated q_rope into dims 512..575
  uint16_t* gate;        // [rows][64]
  uint16_t* q_idx;       // [rows][64][128]
  int splits;
  size_t split_stride;
  RopeFreqs freqs;
};

// Blocks (token, part): q_nope, the rotated q_rope, the gate logits and the
// indexer query.  The token's 32 rotation angles are formed once per block and
// shared by its 64 heads.
__global__ void layer_prep_q_kernel(PrepQArgs a) {
  __shared__ float cs[kRope / 2][2];
  grid_dependency_wait_layer();
  const int row = blockIdx.x;
  const int pos = a.q_pos[row];  // range-checked where the caches are written; only the angle uses it here
  if (threadIdx.x < kRope / 2) rope_cs(pos, a.freqs.f[threadIdx.x], &cs[threadIdx.x][0], &cs[threadIdx.x][1]);
  __syncthreads();
  const Partials g{a.g2 + static_cast<size_t>(row) * kCqRows, a.splits, a.split_stride};
  // items: q_nope (64 x 128) | rope pairs (64 x 32) | gate (64) | q_idx (64 x 128)
  constexpr int kItems = kHeads * kNope + kHeads * (kRope / 2) + kHeads + kIdxHeads * kIdxDim;
  for (int e = blockIdx.y * blockDim.x + threadIdx.x; e < kItems; e += kPrepQParts * blockDim.x) {
    int j = e;
    if (j < kHeads * kNope) {
      const int h = j / kNope, d = j - h * kNope;
      a.q_nope[static_cast<size_t>(row) * kHeads * kNope + j] = bf16_bits(g[h * (kNope + kRope) + d]);
      continue;
    }
    j -= kHeads * kNope;
    if (j < kHeads * (kRope / 2)) {
      const int h = j / (kRope / 2), i = j - h * (kRope / 2);
      const size_t src = static_cast<size_t>(h) * (kNope + kRope) + kNope + 2 * i;
      uint16_t* dst = a.q + (static_cast<size_t>(row) * kHeads + h) * kKvDim + kLatent + 2 * i;
      rope_rotate(g[src], g[src + 1], cs[i][0], cs[i][1], &dst[0], &dst[1]);
      continue;
    }
    j -= kHeads * (kRope / 2);
    if (j < kHeads) {
      a.gate[static_cast<size_t>(row) * kHeads + j] = bf16_bits(g[kQRows + j]);
      continue;
    }
    j -= kHeads;
    a.q_idx[static_cast<size_t>(row) * kIdxHeads * kIdxDim + j] = bf16_bits(g[kQRows + kHeads + j]);
  }
}

// dst[r][c] = bf16(src[r][c]) for r < n_rows, c < n_cols (n_cols a multiple of 4, strides of 4 elements).
__global__ void f32_to_bf16_rows_kernel(const float* src, int src_ld, uint16_t* dst, int dst_ld, int n_rows,
                                        int n_cols) {
  grid_dependency_wait_layer();
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

// y[i] = sum_s part[s][i], in split order (float4 at a time; count a multiple of 4).
__global__ void sum_partials_kernel(const float* part, int splits, size_t stride, float* y, size_t count) {
  grid_dependency_wait_layer();
  const size_t n4 = count / 4;
  for (size_t e = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; e < n4;
       e += static_cast<size_t>(gridDim.x) * blockDim.x) {
    // every split's partial loaded before the first add, then added in split order
    float4 u[kMaxGemmSplits];
#pragma unroll
    for (int s = 0; s < kMaxGemmSplits; ++s)
      u[s] = s < splits ? reinterpret_cast<const float4*>(part + static_cast<size_t>(s) * stride)[e]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    float4 v = u[0];
#pragma unroll
    for (int s = 1; s < kMaxGemmSplits; ++s) {
      if (s < splits) {
        v.x += u[s].x;
        v.y += u[s].y;
        v.z += u[s].z;
        v.w += u[s].w;
      }
    }
    reinterpret_cast<float4*>(y)[e] = v;
  }
}

// Launches `kernel` on `grid` x 256 threads with programmatic dependent launch.
template <class... Params, class... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, cudaStream_t s, Args... args) {
  return sga::host::launch_pdl(kernel, grid, dim3(256), 0, s, args...);
}

cudaError_t launch_convert(const float* src, int src_ld, uint16_t* dst, int dst_ld, int n_rows, int n_cols,
                           cudaStream_t s) {
  const long long total = static_cast<long long>(n_rows) * (n_cols / 4);
  const int blocks = static_cast<int>(std::min<long long>((total + 255) / 256, 148LL * 8));
  return launch_pdl(f32_to_bf16_rows_kernel, dim3(blocks), s, src, src_ld, dst, dst_ld, n_rows, n_cols);
}

// The K splits of the three large GEMMs (G1, G2, G5) for `rows` tokens.
struct Splits {
  int g1, g2, g5;
};
Splits layer_splits(int rows, int d_model, int q_rank) {
  return {sga::gemm_splits(q_rank + kHqExtra, rows, d_model, 1, kSplitSms),
          sga::gemm_splits(kCqRows, rows, q_rank, 1, kSplitSms), sga::gemm_splits(d_model, rows, kOWidth, 1, kSplitSms)};
}

// ---------------------------------------------------------------- workspace
struct LayerLayout {
  size_t path = 0;  // sga_forward's workspace (its status word is the layer's)
  size_t g1 = 0, c_q = 0, g2 = 0, q_nope = 0, q = 0, gate = 0, q_idx = 0, w = 0;
  size_t out = 0, out_b = 0, o_b = 0, y_part = 0, total = 0;
  Splits splits = {1, 1, 1};
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
sga_status_t layer_layout(const sga_dims_t& d, int d_model, int q_rank, sga_layer_op_t op, LayerLayout* l) {
  const size_t rows = static_cast<size_t>(d.batch) * d.n_q;
  l->splits = layer_splits(static_cast<int>(rows), d_model, q_rank);
  size_t off = kStatusBytes;
  if (op == SGA_LAYER_FORWARD) {
    size_t path_bytes = 0;
    if (d.top_k < 64 || d.top_k > SGA_MAX_TOP_K || d.top_k % 64 != 0) return SGA_ERR_INVALID_ARG;
    const sga_status_t st = sga_workspace_size(&d, SGA_OP_FORWARD, &path_bytes);
    if (st != SGA_OK) return st;
    l->path = 0;
    off = align_up(path_bytes);
  }
  if (op != SGA_LAYER_OUTPUT) {
    l->g1 = off;
    off += align_up(l->splits.g1 * rows * (q_rank + kHqExtra) * 4);
    l->c_q = off;
    off += align_up(rows * q_rank * 2);
    l->g2 = off;
    off += align_up(l->splits.g2 * rows * kCqRows * 4);
    l->q_nope = off;
    off += align_up(rows * kHeads * kNope * 2);
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
    l->o_b = off;
    off += align_up(rows * kOWidth * 2);
    l->y_part = off;
    if (l->splits.g5 > 1) off += align_up(l->splits.g5 * rows * static_cast<size_t>(d_model) * 4);
  }
  l->total = off;
  return SGA_OK;
}

bool weights_ok(const sga_layer_weights_t* W, bool front, bool back) {
  if (front && (!aligned(W->w_hq, 16) || !aligned(W->w_cq, 16) || !aligned(W->w_uk, 16))) return false;
  if (back && (!aligned(W->w_uv, 16) || !aligned(W->w_o, 16))) return false;
  return true;
}

// An sm_100 device: its SM count.
sga_status_t device_sms(int* sms) {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  return major == 10 ? SGA_OK : SGA_ERR_UNSUPPORTED;
}

sga_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SGA_OK;
  cudaGetLastError();
  return SGA_ERR_CUDA;
}

// G1, P1, G2, P2, G3: the path's inputs for the new tokens.
sga_status_t project_impl(const sga_dims_t& d, const sga_layer_weights_t* W, const uint16_t* h, const int32_t* q_pos,
                          uint16_t* kv_cache, uint16_t* kidx_cache, uint16_t* q, uint16_t* gate, uint16_t* q_idx,
                          uint16_t* w, void* ws, const LayerLayout& l, int sms, cudaStream_t s) {
  const int rows = d.batch * d.n_q;
  const int R = W->q_rank;
  int* status = at<int>(ws, 0);
  float* g1 = at<float>(ws, l.g1);
  uint16_t* c_q = at<uint16_t>(ws, l.c_q);
  float* g2 = at<float>(ws, l.g2);
  uint16_t* q_nope = at<uint16_t>(ws, l.q_nope);
  cudaError_t e;
  {
    sga::host::NvtxRange range("sga.layer.g1_hq");
    // G1: [rows][R + 768] = h W_hq^T
    sga::GemmArgs ga{W->w_hq, h, R + kHqExtra, rows, W->d_model, 1, false, W->d_model, 0, l.splits.g1, g1,
                     nullptr, 0, 0, status};
    if ((e = sga::launch_gemm(ga, sms, s)) != cudaSuccess) return from_cuda(e);
    PrepHArgs pa{g1, q_pos, c_q, kv_cache, kidx_cache, w, status, R, d.n_q, d.kv_stride, l.splits.g1,
                 static_cast<size_t>(rows) * (R + kHqExtra), rope_freqs()};
    if ((e = launch_pdl(layer_prep_h_kernel, dim3(rows, kPrepHParts), s, pa)) != cudaSuccess) return from_cuda(e);
  }
  {
    sga::host::NvtxRange range("sga.layer.g2_cq");
    // G2: [rows][20544] = c_q W_cq^T
    sga::GemmArgs ga{W->w_cq, c_q, kCqRows, rows, R, 1, false, R, 0, l.splits.g2, g2, nullptr, 0, 0, status};
    if ((e = sga::launch_gemm(ga, sms, s)) != cudaSuccess) return from_cuda(e);
    PrepQArgs qa{g2, q_pos, q_nope, q, gate, q_idx, l.splits.g2, static_cast<size_t>(rows) * kCqRows, rope_freqs()};
    if ((e = launch_pdl(layer_prep_q_kernel, dim3(rows, kPrepQParts), s, qa)) != cudaSuccess) return from_cuda(e);
  }
  sga::host::NvtxRange range("sga.layer.g3_uk");
  // G3: q[r][h][j] = bf16(sum_d W_UK[h][d][j] q_nope[r][h][d]): per head, W_UK[h] is
  // [128 d][512 j] (MN-major in j), the tokens read q_nope's 128 columns of head h
  sga::GemmArgs ga{W->w_uk, q_nope, kLatent, rows, kNope, kHeads, true, kHeads * kNope, kNope, 1, nullptr, q,
                   kHeads * kKvDim, kKvDim, status};
  return from_cuda(sga::launch_gemm(ga, sms, s));
}

// out -> bf16, G4 (W_UV per head, bf16 out), G5 (o_proj) and the sum of its partials.
// With out_b_ready, out_b already holds bf16(out) (written by the attention) and the conversion is skipped.
sga_status_t output_impl(const sga_dims_t& d, const sga_layer_weights_t* W, const float* out, float* y, void* ws,
                         const LayerLayout& l, int sms, cudaStream_t s, bool out_b_ready = false) {
  const int rows = d.batch * d.n_q;
  int* status = at<int>(ws, 0);
  uint16_t* out_b = at<uint16_t>(ws, l.out_b);
  uint16_t* o_b = at<uint16_t>(ws, l.o_b);
  cudaError_t e;
  {
    sga::host::NvtxRange range("sga.layer.g4_uv");
    if (!out_b_ready &&
        (e = launch_convert(out, kLatent, out_b, kLatent, rows * kHeads, kLatent, s)) != cudaSuccess)
      return from_cuda(e);
    // G4: o[r][h][i] = bf16(sum_j W_UV[h][i][j] out[r][h][j]): W_UV[h] is [128 i][512 j] (K-major)
    sga::GemmArgs ga{W->w_uv, out_b, kVHead, rows, kLatent, kHeads, false, kHeads * kLatent, kLatent, 1, nullptr, o_b,
                     kOWidth, kVHead, status};
    if ((e = sga::launch_gemm(ga, sms, s)) != cudaSuccess) return from_cuda(e);
  }
  sga::host::NvtxRange range("sga.layer.g5_o");
  // G5: y = o W_O^T (partials in the workspace when K is split)
  const int s5 = l.splits.g5;
  float* part = s5 > 1 ? at<float>(ws, l.y_part) : y;
  sga::GemmArgs ga{W->w_o, o_b, W->d_model, rows, kOWidth, 1, false, kOWidth, 0, s5, part, nullptr, 0, 0, status};
  if ((e = sga::launch_gemm(ga, sms, s)) != cudaSuccess) return from_cuda(e);
  if (s5 > 1) {
    const size_t count = static_cast<size_t>(rows) * W->d_model;
    const int blocks = static_cast<int>(std::min<size_t>((count / 4 + 255) / 256, 148u * 8));
    if ((e = launch_pdl(sum_partials_kernel, dim3(blocks), s, static_cast<const float*>(part), s5, count, y, count)) !=
        cudaSuccess)
      return from_cuda(e);
  }
  return SGA_OK;
}

sga_status_t check_layer_ws(void* ws, size_t ws_bytes, const sga_dims_t& d, const sga_layer_weights_t* W,
                            sga_layer_op_t op, LayerLayout* l) {
  const sga_status_t st = layer_layout(d, W->d_model, W->q_rank, op, l);
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
  const sga_status_t st = layer_layout(*dims, weights->d_model, weights->q_rank, op, &l);
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
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights, SGA_LAYER_PROJECT, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_sms(&sms)) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return project_impl(*dims, weights, h, q_pos, kv_cache, k_idx_cache, q, gate, q_idx, w, ws, l, sms, s);
}

sga_status_t sga_layer_output(const sga_dims_t* dims, const sga_layer_weights_t* weights, const float* out, float* y,
                              void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!layer_dims_ok(dims, weights) || !weights_ok(weights, false, true)) return SGA_ERR_INVALID_ARG;
  if (!aligned(out, 16) || !aligned(y, 16)) return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights, SGA_LAYER_OUTPUT, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_sms(&sms)) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return output_impl(*dims, weights, out, y, ws, l, sms, s);
}

sga_status_t sga_layer_forward(const sga_dims_t* dims, const sga_layer_weights_t* weights, const sga_bf16_t* h,
                               const int32_t* q_pos, sga_bf16_t* kv_cache, sga_bf16_t* k_idx_cache, int32_t* idx_out,
                               float* y, void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!layer_dims_ok(dims, weights) || !weights_ok(weights, true, true)) return SGA_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(q_pos, 4) || !aligned(kv_cache, 16) || !aligned(k_idx_cache, 16) ||
      !aligned(y, 16) || (idx_out && !aligned(idx_out, 16)))
    return SGA_ERR_INVALID_ARG;
  LayerLayout l;
  sga_status_t st = check_layer_ws(ws, ws_bytes, *dims, weights, SGA_LAYER_FORWARD, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_sms(&sms)) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint16_t* q = at<uint16_t>(ws, l.q);
  uint16_t* gate = at<uint16_t>(ws, l.gate);
  uint16_t* q_idx = at<uint16_t>(ws, l.q_idx);
  uint16_t* w = at<uint16_t>(ws, l.w);
  float* out = at<float>(ws, l.out);
  st = project_impl(*dims, weights, h, q_pos, kv_cache, k_idx_cache, q, gate, q_idx, w, ws, l, sms, s);
  if (st != SGA_OK) return st;
  size_t path_bytes = 0;
  sga_workspace_size(dims, SGA_OP_FORWARD, &path_bytes);
  // the attention also writes its output in bf16 for W_UV: no conversion pass
  st = sga::forward_bf16_copy(dims, q_idx, w, k_idx_cache, q, kv_cache, gate, q_pos, idx_out, out,
                              at<uint16_t>(ws, l.out_b), ws, path_bytes, stream);
  if (st != SGA_OK) return st;
  return output_impl(*dims, weights, out, y, ws, l, sms, s, true);
}

}  // extern "C"
