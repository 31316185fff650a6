// The indexer's sparse warm-up objective and its gradients (arXiv abstract
// "A.X K2 Technical Report": the indexer is optimised against its own sparse
// top-k selection rather than the dense attention distribution; archdb
// "A.X K2", stage notes: indexer-only training with the backbone frozen).
// The pages give no formula; the reading (DSA style), for query t with its
// selection S (the idx the path returns):
//
//   p(s) = (1/64) sum_h softmax_{s in S}((q_h . kv_s) * 192^-0.5)   frozen target, no gradient
//   r(s) = softmax_{s in S}(score(s)),  score(s) = sum_j w_j ReLU(a_js),  a_js = q_idx_j . k_idx_s
//   loss = KL(p || r) = sum_{s in S} p(s) (log p(s) - log r(s))
//   g_s = r(s) - p(s)
//   dw_j = sum_s g_s ReLU(a_js)
//   dq_idx_j = sum_s g_s w_j [a_js > 0] k_idx_s
//   dk_idx_s += sum_j g_s w_j [a_js > 0] q_idx_j        (summed over the queries that select s)
//
// Three kernels, all plain fp32 SIMT arithmetic on bf16 inputs:
//   A  per (query, 64-slot chunk): gathers the chunk's latent and key rows,
//      writes the 64 head logits z, the 64 indexer dots a and the score of
//      every slot to the workspace (empty slots: z = -inf);
//   B  per query: per-head softmax statistics, the target p, the indexer
//      softmax r, the loss and g = r - p; zeroes the query's q_idx and w
//      gradients;
//   C  per (query, chunk): accumulates the gradients with atomic adds.
// Staged rows are padded by 16 bytes so that the rows a warp reads at once
// start on different shared-memory banks.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sga.h"
#include "sga_host.h"

namespace {

constexpr int kHeads = SGA_HEADS;           // 64
constexpr int kDq = SGA_QK_DIM;             // 576
constexpr int kIdxHeads = SGA_INDEX_HEADS;  // 64
constexpr int kIdxDim = SGA_INDEX_DIM;      // 128
constexpr int kChunk = 64;                  // selected slots per CTA
constexpr int kThreads = 256;
constexpr int kRowPad = kDq + 8;            // staged q / kv row: 584 bf16 (1168 B)
constexpr int kIdxPad = kIdxDim + 8;        // staged q_idx / k_idx row: 136 bf16 (272 B)
constexpr float kScale = static_cast<float>(SGA_SOFTMAX_SCALE);
using sga::host::align_up;
using sga::host::aligned;
using sga::host::at;
using sga::host::kStatusBytes;
constexpr size_t kAlign = sga::host::kWsAlign;

// kernel A: q, kv rows, q_idx, k rows (bf16, padded), a (fp32)
constexpr size_t kLogitsSmem = (2 * kHeads * kRowPad + 2 * kChunk * kIdxPad) * 2 + kIdxHeads * kChunk * 4;
// kernel C: q_idx, k rows (bf16, padded), act and ReLU(a) (fp32)
constexpr size_t kGradSmem = 2 * kChunk * kIdxPad * 2 + 2 * kIdxHeads * kChunk * 4;
static_assert(kLogitsSmem <= 232448 && kGradSmem <= 232448, "shared memory");

struct WarmupArgs {
  const uint16_t* q_idx;  // [rows][64][128]
  const uint16_t* w;      // [rows][64]
  const uint16_t* k_idx;  // [B][L][128]
  const uint16_t* q;      // [rows][64][576]
  const uint16_t* kv;     // [B][L][576]
  const int32_t* idx;     // [rows][K]
  float* loss;            // [rows]
  float* grad_q_idx;      // [rows][64][128]
  float* grad_w;          // [rows][64]
  float* grad_k_idx;      // [B][L][128], accumulated
  float* z;               // workspace [rows][64][K]
  float* a;               // workspace [rows][64][K]
  float* score;           // workspace [rows][K]
  float* g;               // workspace [rows][K]
  int* status;
  int n_q, kv_stride, top_k;
};

__device__ __forceinline__ float bf(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Block-wide reduction (kThreads threads); `red` holds kThreads / 32 floats.
template <bool kMax>
__device__ float block_reduce(float v, float* red) {
  v = kMax ? warp_max(v) : warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = lane < kThreads / 32 ? red[lane] : (kMax ? -INFINITY : 0.f);
  return kMax ? warp_max(v) : warp_sum(v);
}

// The cache row of each slot of the chunk (-1: empty); out-of-range indices are recorded and dropped.
__device__ void load_slot_rows(const WarmupArgs& p, int row, int c, int* slot_row) {
  const int t = threadIdx.x;
  if (t < kChunk) {
    int s = p.idx[static_cast<size_t>(row) * p.top_k + static_cast<size_t>(c) * kChunk + t];
    if (s < -1 || s >= p.kv_stride) {
      atomicCAS(p.status, 0, static_cast<int>(SGA_ERR_DEVICE_ARG));
      s = -1;
    }
    slot_row[t] = s;
  }
}

// Copies `rows` rows of `width` bf16 (16-byte aligned, width a multiple of 8) into padded shared rows.
__device__ void stage_rows(uint16_t* dst, int pad, const uint16_t* src, int width, int rows) {
  const int vecs = width / 8;
  for (int e = threadIdx.x; e < rows * vecs; e += kThreads) {
    const int r = e / vecs, v = e - r * vecs;
    *reinterpret_cast<uint4*>(dst + r * pad + v * 8) =
        reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * width)[v];
  }
}

// Gathers the chunk's cache rows (zeros for empty slots) into padded shared rows.
__device__ void gather_rows(uint16_t* dst, int pad, const uint16_t* cache, int width, size_t seq_base,
                            const int* slot_row) {
  const int vecs = width / 8;
  for (int e = threadIdx.x; e < kChunk * vecs; e += kThreads) {
    const int s = e / vecs, v = e - s * vecs;
    const int r = slot_row[s];
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r >= 0) val = reinterpret_cast<const uint4*>(cache + (seq_base + r) * width)[v];
    *reinterpret_cast<uint4*>(dst + s * pad + v * 8) = val;
  }
}

// A: logits, indexer dots and scores of one chunk of selected slots.
__global__ void __launch_bounds__(kThreads) warmup_logits_kernel(WarmupArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* qs = reinterpret_cast<uint16_t*>(smem);  // [64][kRowPad]
  uint16_t* kvs = qs + kHeads * kRowPad;               // [64][kRowPad]
  uint16_t* qis = kvs + kChunk * kRowPad;              // [64][kIdxPad]
  uint16_t* ks = qis + kIdxHeads * kIdxPad;            // [64][kIdxPad]
  float* as = reinterpret_cast<float*>(ks + kChunk * kIdxPad);  // [64 j][64 s]
  __shared__ int slot_row[kChunk];
  const int c = blockIdx.x, row = blockIdx.y, b = row / p.n_q, t = threadIdx.x;
  const size_t seq_base = static_cast<size_t>(b) * p.kv_stride;
  load_slot_rows(p, row, c, slot_row);
  stage_rows(qs, kRowPad, p.q + static_cast<size_t>(row) * kHeads * kDq, kDq, kHeads);
  stage_rows(qis, kIdxPad, p.q_idx + static_cast<size_t>(row) * kIdxHeads * kIdxDim, kIdxDim, kIdxHeads);
  __syncthreads();
  gather_rows(kvs, kRowPad, p.kv, kDq, seq_base, slot_row);
  gather_rows(ks, kIdxPad, p.k_idx, kIdxDim, seq_base, slot_row);
  __syncthreads();
  const int h = t >> 2, s0 = t & 3;  // head (or indexer head) and first slot of this thread
  {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    const __nv_bfloat162* qh = reinterpret_cast<const __nv_bfloat162*>(qs + h * kRowPad);
    for (int d2 = 0; d2 < kDq / 2; ++d2) {
      const float2 qv = __bfloat1622float2(qh[d2]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 kv2 =
            __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(kvs + (s0 + 4 * i) * kRowPad)[d2]);
        acc[i] = fmaf(qv.x, kv2.x, acc[i]);
        acc[i] = fmaf(qv.y, kv2.y, acc[i]);
      }
    }
    float* zr = p.z + (static_cast<size_t>(row) * kHeads + h) * p.top_k + static_cast<size_t>(c) * kChunk;
#pragma unroll
    for (int i = 0; i < 16; ++i) zr[s0 + 4 * i] = slot_row[s0 + 4 * i] >= 0 ? acc[i] * kScale : -INFINITY;
  }
  {
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    const __nv_bfloat162* qj = reinterpret_cast<const __nv_bfloat162*>(qis + h * kIdxPad);
    for (int d2 = 0; d2 < kIdxDim / 2; ++d2) {
      const float2 qv = __bfloat1622float2(qj[d2]);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 k2 = __bfloat1622float2(reinterpret_cast<const __nv_bfloat162*>(ks + (s0 + 4 * i) * kIdxPad)[d2]);
        acc[i] = fmaf(qv.x, k2.x, acc[i]);
        acc[i] = fmaf(qv.y, k2.y, acc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) as[h * kChunk + s0 + 4 * i] = acc[i];
  }
  __syncthreads();
  for (int e = t; e < kIdxHeads * kChunk; e += kThreads) {
    const int j = e / kChunk, s = e - j * kChunk;
    p.a[(static_cast<size_t>(row) * kIdxHeads + j) * p.top_k + static_cast<size_t>(c) * kChunk + s] = as[e];
  }
  if (t < kChunk) {
    float sc = 0.f;
    for (int j = 0; j < kIdxHeads; ++j)
      sc = fmaf(bf(p.w[static_cast<size_t>(row) * kIdxHeads + j]), fmaxf(as[j * kChunk + t], 0.f), sc);
    p.score[static_cast<size_t>(row) * p.top_k + static_cast<size_t>(c) * kChunk + t] = sc;
  }
}

// B: per query, the target p, the indexer softmax r, the loss and g = r - p.
__global__ void __launch_bounds__(kThreads) warmup_objective_kernel(WarmupArgs p) {
  __shared__ float hm[kHeads], hl[kHeads], red[kThreads / 32];
  const int row = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int K = p.top_k;
  const float* zr = p.z + static_cast<size_t>(row) * kHeads * K;
  const float* sr = p.score + static_cast<size_t>(row) * K;
  for (int h = warp; h < kHeads; h += kThreads / 32) {
    float m = -INFINITY;
    for (int s = lane; s < K; s += 32) m = fmaxf(m, zr[static_cast<size_t>(h) * K + s]);
    m = warp_max(m);
    float l = 0.f;
    if (m != -INFINITY)
      for (int s = lane; s < K; s += 32) l += expf(zr[static_cast<size_t>(h) * K + s] - m);
    l = warp_sum(l);
    if (lane == 0) {
      hm[h] = m;
      hl[h] = l;
    }
  }
  // the indexer softmax over the valid slots (an empty slot has z = -inf in every head)
  float smax = -INFINITY;
  for (int s = t; s < K; s += kThreads)
    if (zr[s] != -INFINITY) smax = fmaxf(smax, sr[s]);
  smax = block_reduce<true>(smax, red);
  float ssum = 0.f;
  if (smax != -INFINITY)
    for (int s = t; s < K; s += kThreads)
      if (zr[s] != -INFINITY) ssum += expf(sr[s] - smax);
  ssum = block_reduce<false>(ssum, red);
  const float log_ssum = logf(ssum);
  float part = 0.f;
  for (int s = t; s < K; s += kThreads) {
    float gs = 0.f;
    if (zr[s] != -INFINITY) {
      float pp = 0.f;
      for (int h = 0; h < kHeads; ++h) pp += expf(zr[static_cast<size_t>(h) * K + s] - hm[h]) / hl[h];
      pp *= 1.f / kHeads;
      const float log_r = sr[s] - smax - log_ssum;
      if (pp > 0.f) part += pp * (logf(pp) - log_r);
      gs = expf(log_r) - pp;
    }
    p.g[static_cast<size_t>(row) * K + s] = gs;
  }
  part = block_reduce<false>(part, red);
  if (t == 0) p.loss[row] = part;
  for (int e = t; e < kIdxHeads * kIdxDim; e += kThreads)
    p.grad_q_idx[static_cast<size_t>(row) * kIdxHeads * kIdxDim + e] = 0.f;
  if (t < kIdxHeads) p.grad_w[static_cast<size_t>(row) * kIdxHeads + t] = 0.f;
}

// C: the gradients of one chunk, added into the query's q_idx and w gradients
// and into the key gradients of the selected cache rows.
__global__ void __launch_bounds__(kThreads) warmup_grad_kernel(WarmupArgs p) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* qis = reinterpret_cast<uint16_t*>(smem);             // [64][kIdxPad]
  uint16_t* ks = qis + kIdxHeads * kIdxPad;                        // [64][kIdxPad]
  float* act = reinterpret_cast<float*>(ks + kChunk * kIdxPad);   // [64 j][64 s]: g_s w_j [a_js > 0]
  float* relu = act + kIdxHeads * kChunk;                          // [64 j][64 s]: ReLU(a_js)
  __shared__ int slot_row[kChunk];
  __shared__ float gs[kChunk], wj[kIdxHeads];
  const int c = blockIdx.x, row = blockIdx.y, b = row / p.n_q, t = threadIdx.x;
  const size_t seq_base = static_cast<size_t>(b) * p.kv_stride;
  load_slot_rows(p, row, c, slot_row);
  if (t < kChunk) gs[t] = p.g[static_cast<size_t>(row) * p.top_k + static_cast<size_t>(c) * kChunk + t];
  if (t < kIdxHeads) wj[t] = bf(p.w[static_cast<size_t>(row) * kIdxHeads + t]);
  stage_rows(qis, kIdxPad, p.q_idx + static_cast<size_t>(row) * kIdxHeads * kIdxDim, kIdxDim, kIdxHeads);
  __syncthreads();
  gather_rows(ks, kIdxPad, p.k_idx, kIdxDim, seq_base, slot_row);
  for (int e = t; e < kIdxHeads * kChunk; e += kThreads) {
    const int j = e / kChunk, s = e - j * kChunk;
    const float av =
        p.a[(static_cast<size_t>(row) * kIdxHeads + j) * p.top_k + static_cast<size_t>(c) * kChunk + s];
    const bool on = slot_row[s] >= 0 && av > 0.f;
    act[e] = on ? gs[s] * wj[j] : 0.f;
    relu[e] = on ? av : 0.f;
  }
  __syncthreads();
  if (t < kIdxHeads) {
    float acc = 0.f;
    for (int s = 0; s < kChunk; ++s) acc = fmaf(gs[s], relu[t * kChunk + s], acc);
    atomicAdd(&p.grad_w[static_cast<size_t>(row) * kIdxHeads + t], acc);
  }
  const int q4 = t >> 2, d0 = (t & 3) * 32;
  {
    // dq_idx[j][d0 .. d0+31], j = q4
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;
    for (int s = 0; s < kChunk; ++s) {
      const float av = act[q4 * kChunk + s];
      const __nv_bfloat162* kr = reinterpret_cast<const __nv_bfloat162*>(ks + s * kIdxPad + d0);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 k2 = __bfloat1622float2(kr[i]);
        acc[2 * i] = fmaf(av, k2.x, acc[2 * i]);
        acc[2 * i + 1] = fmaf(av, k2.y, acc[2 * i + 1]);
      }
    }
    float* dst = p.grad_q_idx + (static_cast<size_t>(row) * kIdxHeads + q4) * kIdxDim + d0;
#pragma unroll
    for (int i = 0; i < 32; ++i) atomicAdd(dst + i, acc[i]);
  }
  {
    // dk[s][d0 .. d0+31], s = q4
    const int r = slot_row[q4];
    if (r >= 0) {
      float acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = 0.f;
      for (int j = 0; j < kIdxHeads; ++j) {
        const float av = act[j * kChunk + q4];
        const __nv_bfloat162* qr = reinterpret_cast<const __nv_bfloat162*>(qis + j * kIdxPad + d0);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 q2 = __bfloat1622float2(qr[i]);
          acc[2 * i] = fmaf(av, q2.x, acc[2 * i]);
          acc[2 * i + 1] = fmaf(av, q2.y, acc[2 * i + 1]);
        }
      }
      float* dst = p.grad_k_idx + (seq_base + r) * kIdxDim + d0;
#pragma unroll
      for (int i = 0; i < 32; ++i) atomicAdd(dst + i, acc[i]);
    }
  }
}


struct WarmupLayout {
  size_t z = 0, a = 0, score = 0, g = 0, total = 0;
};

bool warmup_dims_ok(const sga_dims_t* d) {
  if (!d || d->batch < 1 || d->n_q < 1 || d->kv_stride < 1 || d->kv_stride > SGA_MAX_KV_STRIDE) return false;
  if (d->top_k < kChunk || d->top_k > SGA_MAX_TOP_K || d->top_k % kChunk != 0) return false;
  const long long rows = static_cast<long long>(d->batch) * d->n_q;
  return rows <= 65535 && static_cast<long long>(d->batch) * d->kv_stride <= INT32_MAX;
}

WarmupLayout warmup_layout(const sga_dims_t& d) {
  WarmupLayout l;
  const size_t rows = static_cast<size_t>(d.batch) * d.n_q, K = static_cast<size_t>(d.top_k);
  size_t off = kStatusBytes;
  l.z = off;
  off += align_up(rows * kHeads * K * 4);
  l.a = off;
  off += align_up(rows * kIdxHeads * K * 4);
  l.score = off;
  off += align_up(rows * K * 4);
  l.g = off;
  off += align_up(rows * K * 4);
  l.total = off;
  return l;
}

}  // namespace

extern "C" {

sga_status_t sga_indexer_warmup_workspace_size(const sga_dims_t* dims, size_t* bytes) {
  if (!bytes || !warmup_dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  *bytes = warmup_layout(*dims).total;
  return SGA_OK;
}

sga_status_t sga_indexer_warmup(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                                const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                                const int32_t* idx, float* loss, float* grad_q_idx, float* grad_w, float* grad_k_idx,
                                void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!warmup_dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(w, 2) || !aligned(k_idx, 16) || !aligned(q, 16) || !aligned(kv, 16) ||
      !aligned(idx, 4) || !aligned(loss, 4) || !aligned(grad_q_idx, 4) || !aligned(grad_w, 4) ||
      !aligned(grad_k_idx, 4))
    return SGA_ERR_INVALID_ARG;
  const WarmupLayout l = warmup_layout(*dims);
  if (!aligned(ws, kAlign) || ws_bytes < l.total) return SGA_ERR_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  {
    // the kernels' dynamic shared memory limits, set once per device
    static std::mutex mu;
    static bool attrs_set[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= 64) return SGA_ERR_UNSUPPORTED;
    if (!attrs_set[dev]) {
      if (cudaFuncSetAttribute(warmup_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kLogitsSmem)) != cudaSuccess ||
          cudaFuncSetAttribute(warmup_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kGradSmem)) != cudaSuccess)
        return SGA_ERR_CUDA;
      attrs_set[dev] = true;
    }
  }
  WarmupArgs a{q_idx, w, k_idx, q, kv, idx, loss, grad_q_idx, grad_w, grad_k_idx, at<float>(ws, l.z),
               at<float>(ws, l.a), at<float>(ws, l.score), at<float>(ws, l.g), at<int>(ws, 0), dims->n_q,
               dims->kv_stride, dims->top_k};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = dims->batch * dims->n_q;
  const dim3 grid(dims->top_k / kChunk, rows);
  warmup_logits_kernel<<<grid, kThreads, kLogitsSmem, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SGA_ERR_CUDA;
  warmup_objective_kernel<<<rows, kThreads, 0, s>>>(a);
  if (cudaGetLastError() != cudaSuccess) return SGA_ERR_CUDA;
  warmup_grad_kernel<<<grid, kThreads, kGradSmem, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? SGA_OK : SGA_ERR_CUDA;
}

}  // extern "C"
