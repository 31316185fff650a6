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
// Kernels, in launch order:
//   B  per query: clears the query's q_idx and w gradients;
//   A  per (query, 64-slot chunk), on the tensor core: gathers the chunk's
//      latent and key rows, writes the 64 head logits z, the 64 indexer dots
//      a, the score of every slot (empty slots: z = -inf), each head's
//      (max, sum of exponentials) over the chunk and the same pair for the
//      chunk's scores to the workspace;
//   C  per (query, chunk): the target's per-head statistics and the indexer
//      softmax's normaliser, merged from the chunks' pairs; p, r, g = r - p
//      and the loss terms of the chunk's slots; then the gradients, on the
//      tensor core, added with atomics;
//   B  per query: the loss, the chunks' terms summed in chunk order.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sga.h"
#include "sga_host.h"
#include "sga_ptx.cuh"

namespace {

constexpr int kHeads = SGA_HEADS;           // 64
constexpr int kDq = SGA_QK_DIM;             // 576
constexpr int kIdxHeads = SGA_INDEX_HEADS;  // 64
constexpr int kIdxDim = SGA_INDEX_DIM;      // 128
constexpr int kChunk = 64;                  // selected slots per CTA
constexpr int kThreads = 256;
constexpr float kScale = static_cast<float>(SGA_SOFTMAX_SCALE);
using sga::host::align_up;
using sga::host::aligned;
using sga::host::at;
using sga::host::kStatusBytes;
using sga::host::launch_pdl;
constexpr size_t kAlign = sga::host::kWsAlign;

// kernel A (tensor core): 10 swizzled boxes of 64 rows x 64 bf16, and the 1 KB alignment
constexpr int kLogitThreads = 128;
constexpr int kBox = 64 * 128;
constexpr uint32_t kLogitTmemCols = 128;  // z at column 0, a at column 64
constexpr int kLogitPhases = 3;  // Q and the latent rows: three 192-dim phases
constexpr size_t kLogitsSmem = 1024 + 10 * kBox;
// kernel C (tensor core): q_idx, the key rows and act's two parts in six boxes; the request
// is sized so that at most two CTAs (256 tensor-memory columns each) share an SM
constexpr uint32_t kGradTmemCols = 256;  // dq_idx at column 0, dk at column 128
constexpr size_t kGradSmem = 80 * 1024;
static_assert(kGradSmem >= 1024 + 6 * kBox && 3 * (kGradSmem + 4096) > 232448, "two CTAs per SM");
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
  float* loss_part;       // workspace [rows][K / 64]: each chunk's share of the loss
  float2* stats;          // workspace [rows][64][K / 64]: each chunk's (max z, sum exp(z - max)) per head
  float2* score_stats;    // workspace [rows][K / 64]: each chunk's (max score, sum exp(score - max)) over its valid slots
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

// A: logits, indexer dots, scores and the chunk's softmax statistics of one
// chunk of 64 selected slots, on the tensor core.  All 128 threads gather the
// query's 64 x 576 latent query and the chunk's 64 latent rows (in three
// 192-dim phases), the 64 x 128 indexer query and the chunk's 64 key rows into
// 128-byte-swizzled boxes of 64 rows x 64 dims (16-byte cp.async; empty slots
// are zero-filled); one thread issues z = Q C^T (M = 64 heads, N = 64 slots,
// K = 576, accumulated over the phases) and a = Q_idx K^T
// (M = 64 indexer heads, K = 128) into tensor memory; each warp then reads 16
// rows of both with the 16-lane x 256-bit shape (thread t: rows t/4 and 8 + t/4
// of its quarter, columns 8k + 2(t%4) and +1).
__global__ void __launch_bounds__(kLogitThreads, 2) warmup_logits_kernel(WarmupArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // Q and the latent rows arrive in three phases of three 64-dim boxes each
  // (the K = 576 contraction accumulates across them), so one CTA holds 80 KB
  // and two share an SM: one's gathers overlap the other's MMAs and epilogue.
  const uint32_t q_s = sga::smem_u32(smem);    // 3 boxes: the query's 64 heads x 192 dims of this phase
  const uint32_t kv_s = q_s + 3 * kBox;         // 3 boxes: the chunk's 64 latent rows, same dims
  const uint32_t qi_s = kv_s + 3 * kBox;        // 2 boxes: 64 indexer heads x 128
  const uint32_t ki_s = qi_s + 2 * kBox;        // 2 boxes: the chunk's 64 key rows
  __shared__ int slot_row[kChunk];
  __shared__ float sc_part[4][kChunk];
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int c = blockIdx.x, row = blockIdx.y, b = row / p.n_q, t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const size_t seq_base = static_cast<size_t>(b) * p.kv_stride;
  const int nch = p.top_k / kChunk;
  if (t == 0) {
    sga::mbar_init(sga::smem_u32(&mma_bar), 1);
    abort_flag = 0;
    sga::fence_barrier_init();
  }
  if (warp == 0) {
    sga::tmem_alloc(sga::smem_u32(&tmem_slot), kLogitTmemCols);
    sga::tmem_relinquish();
  }
  load_slot_rows(p, row, c, slot_row);
  sga::tc_fence_before();
  __syncthreads();
  sga::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // This kernel reads only the caller's inputs, and its writes go to regions
  // whose last reader (the previous call's kernel C) finished before this grid
  // could start; its tensor memory is held, so kernel C may be scheduled now.
  sga::grid_launch_dependents();
  const uint16_t* qrow = p.q + static_cast<size_t>(row) * kHeads * kDq;
  bool ok = true;
  int committed = 0;  // MMA batches committed to mma_bar
  for (int ph = 0; ph < kLogitPhases && ok; ++ph) {
    if (ph > 0) {
      // the previous phase's MMAs have read the buffers before they are refilled
      ok = sga::mbar_wait(sga::smem_u32(&mma_bar), static_cast<uint32_t>((ph - 1) & 1), &abort_flag);
      if (!ok) {
        atomicCAS(p.status, 0, static_cast<int>(SGA_ERR_TIMEOUT));
        abort_flag = 1;
      }
      ok = __syncthreads_and(ok) != 0;
      if (!ok) break;
      sga::tc_fence_after();
    }
    // 16-byte pieces: this phase's 24 of a 576-wide row's 72 (box (piece >> 3) % 3, part piece & 7)
    for (int e = t; e < kHeads * 24; e += kLogitThreads) {
      const int r = e / 24, pc = e - r * 24, gp = 24 * ph + pc;
      sga::cp_async_16(q_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4), qrow + r * kDq + gp * 8, 16);
    }
    for (int e = t; e < kChunk * 24; e += kLogitThreads) {
      const int r = e / 24, pc = e - r * 24, gp = 24 * ph + pc, sr = slot_row[r];
      const uint16_t* src = p.kv + (seq_base + (sr >= 0 ? sr : 0)) * kDq + gp * 8;
      sga::cp_async_16(kv_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4), src, sr >= 0 ? 16u : 0u);
    }
    if (ph == 0) {
      const uint16_t* qirow = p.q_idx + static_cast<size_t>(row) * kIdxHeads * kIdxDim;
      for (int e = t; e < kIdxHeads * 16; e += kLogitThreads) {
        const int r = e >> 4, pc = e & 15;
        sga::cp_async_16(qi_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4),
                         qirow + r * kIdxDim + pc * 8, 16);
      }
      for (int e = t; e < kChunk * 16; e += kLogitThreads) {
        const int r = e >> 4, pc = e & 15, sr = slot_row[r];
        const uint16_t* src = p.k_idx + (seq_base + (sr >= 0 ? sr : 0)) * kIdxDim + pc * 8;
        sga::cp_async_16(ki_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4), src, sr >= 0 ? 16u : 0u);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    sga::fence_proxy_async_smem();  // written by cp.async, read by the tensor core
    __syncthreads();
    if (t == 0) {
      constexpr uint32_t idesc = sga::idesc_bf16_f32(kHeads, kChunk, false, false);
      sga::tc_fence_after();
      for (int bx = 0; bx < 3; ++bx)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          sga::mma_bf16(tmem, sga::sdesc_sw128(q_s + bx * kBox + kk * 32, 16, 1024),
                        sga::sdesc_sw128(kv_s + bx * kBox + kk * 32, 16, 1024), idesc, (ph | bx | kk) ? 1u : 0u);
      if (ph == 0) {
        for (int bx = 0; bx < 2; ++bx)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            sga::mma_bf16(tmem + kChunk, sga::sdesc_sw128(qi_s + bx * kBox + kk * 32, 16, 1024),
                          sga::sdesc_sw128(ki_s + bx * kBox + kk * 32, 16, 1024), idesc, (bx | kk) ? 1u : 0u);
      }
      sga::mma_commit(sga::smem_u32(&mma_bar));
    }
    ++committed;
  }
  if (ok) {
    ok = sga::mbar_wait(sga::smem_u32(&mma_bar), static_cast<uint32_t>((committed - 1) & 1), &abort_flag);
    if (!ok) {
      atomicCAS(p.status, 0, static_cast<int>(SGA_ERR_TIMEOUT));
      abort_flag = 1;
    }
    ok = __syncthreads_and(ok) != 0;  // the epilogue's shuffles need whole warps
  }
  sga::tc_fence_after();
  if (ok) {
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    float r[32], ra[32];
    sga::tmem_ld_16x256b_x8(tmem + lane_addr, r);
    sga::tmem_ld_16x256b_x8(tmem + lane_addr + kChunk, ra);
    const int m4 = lane & 3;
    const int hr[2] = {warp * 16 + (lane >> 2), warp * 16 + 8 + (lane >> 2)};  // this thread's two rows
    const float wj[2] = {bf(p.w[static_cast<size_t>(row) * kIdxHeads + hr[0]]),
                         bf(p.w[static_cast<size_t>(row) * kIdxHeads + hr[1]])};
    float sc[16];  // this thread's score partials, columns 8k + 2 m4 + e
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      float zz[16];
      float m = -INFINITY;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = 8 * k + 2 * m4 + e;
          zz[2 * k + e] = slot_row[col] >= 0 ? r[4 * k + 2 * i + e] * kScale : -INFINITY;
          m = fmaxf(m, zz[2 * k + e]);
        }
      }
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
      float l = 0.f;
      if (m != -INFINITY) {
#pragma unroll
        for (int k = 0; k < 16; ++k) l += expf(zz[k] - m);
      }
      l += __shfl_xor_sync(0xffffffffu, l, 1);
      l += __shfl_xor_sync(0xffffffffu, l, 2);
      const size_t zrow = (static_cast<size_t>(row) * kHeads + hr[i]) * p.top_k + static_cast<size_t>(c) * kChunk;
      const size_t arow = (static_cast<size_t>(row) * kIdxHeads + hr[i]) * p.top_k + static_cast<size_t>(c) * kChunk;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int col = 8 * k + 2 * m4;
        *reinterpret_cast<float2*>(p.z + zrow + col) = make_float2(zz[2 * k], zz[2 * k + 1]);
        *reinterpret_cast<float2*>(p.a + arow + col) = make_float2(ra[4 * k + 2 * i], ra[4 * k + 2 * i + 1]);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float v = wj[i] * fmaxf(ra[4 * k + 2 * i + e], 0.f);
          sc[2 * k + e] = i == 0 ? v : sc[2 * k + e] + v;
        }
      }
      if (m4 == 0)
        p.stats[(static_cast<size_t>(row) * kHeads + hr[i]) * nch + c] = make_float2(m, l);
    }
    // the warp's 16 rows summed (lanes that share m4 hold the same columns)
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      sc[k] += __shfl_xor_sync(0xffffffffu, sc[k], 4);
      sc[k] += __shfl_xor_sync(0xffffffffu, sc[k], 8);
      sc[k] += __shfl_xor_sync(0xffffffffu, sc[k], 16);
    }
    if (lane < 4) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        sc_part[warp][8 * k + 2 * m4] = sc[2 * k];
        sc_part[warp][8 * k + 2 * m4 + 1] = sc[2 * k + 1];
      }
    }
  } else if (t == 0 && committed > 0) {
    volatile int never = 0;  // the last committed batch's MMAs must finish before tensor memory is freed
    sga::mbar_wait(sga::smem_u32(&mma_bar), static_cast<uint32_t>((committed - 1) & 1), &never);
  }
  sga::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sga::tc_fence_after();
    sga::tmem_dealloc(tmem, kLogitTmemCols);
  }
  // the score of slot t (warps 0 and 1), and the chunk's (max, sum of exponentials) over its valid slots
  __shared__ float smax_w[2], ssum_w[2];
  float sc = 0.f;
  const bool valid = t < kChunk && slot_row[t] >= 0;
  if (t < kChunk) {
    sc = (sc_part[0][t] + sc_part[1][t]) + (sc_part[2][t] + sc_part[3][t]);
    if (ok) p.score[static_cast<size_t>(row) * p.top_k + static_cast<size_t>(c) * kChunk + t] = sc;
    const float m = warp_max(valid ? sc : -INFINITY);
    if (lane == 0) smax_w[warp] = m;
  }
  __syncthreads();
  const float cmax = fmaxf(smax_w[0], smax_w[1]);
  if (t < kChunk) {
    const float e = warp_sum(valid && cmax != -INFINITY ? expf(sc - cmax) : 0.f);
    if (lane == 0) ssum_w[warp] = e;
  }
  __syncthreads();
  if (ok && t == 0) p.score_stats[static_cast<size_t>(row) * nch + c] = make_float2(cmax, ssum_w[0] + ssum_w[1]);
  // not done before the first kernel B is: kernel C, which waits for this
  // grid, adds into the gradients that kernel B clears
  sga::grid_dependency_wait();
}

// C: per (query, chunk), the objective for the chunk's slots, then their
// gradients.  The target's per-head statistics and the indexer softmax's
// normaliser come merged from every chunk's (max, sum) pairs; then for each
// slot p(s), r(s), g_s = r(s) - p(s) and its loss term
// (the chunk's share goes to the workspace, summed in chunk order by kernel
// B).  With act[j][s] = g_s w_j [a_js > 0], carried as two bf16 parts (hi +
// lo, about 16 mantissa bits), the tensor core computes
//   dq_idx[j][d] = sum_s act[j][s] k[s][d]   (M = 64 j, N = 128 d, K = 64 s;
//                                              act K-major, k rows MN-major)
//   dk[s][d]     = sum_j act[j][s] q_idx[j][d] (M = 64 s, N = 128 d, K = 64 j;
//                                              act and q_idx MN-major)
// into tensor memory (columns 0 and 128); eight warps read them back (warps
// 0-3 dq_idx, 4-7 dk, one TMEM lane quarter each) and add them to the query's
// q_idx gradient and the selected rows' key gradients with float2 atomics.
// dw_j = sum_s g_s ReLU(a_js) is summed by the threads that build act.
__global__ void __launch_bounds__(kThreads, 2) warmup_grad_kernel(WarmupArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t qi_s = sga::smem_u32(smem);  // 2 boxes: q_idx [64 j][128 d]
  const uint32_t ki_s = qi_s + 2 * kBox;       // 2 boxes: the chunk's key rows [64 s][128 d]
  const uint32_t ah_s = ki_s + 2 * kBox;       // act, high bf16 part [64 j][64 s]
  const uint32_t al_s = ah_s + kBox;           // act, low part
  uint8_t* ah_ptr = smem + 4 * kBox;
  __shared__ int slot_row[kChunk];
  __shared__ float gs[kChunk], wj[kIdxHeads], hm[kHeads], hinv[kHeads], red[kThreads / 32];
  __shared__ float pp_part[kThreads / kChunk][kChunk];
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int c = blockIdx.x, row = blockIdx.y, b = row / p.n_q, t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  const int K = p.top_k, nch = K / kChunk;
  const size_t seq_base = static_cast<size_t>(b) * p.kv_stride;
  if (t == 0) {
    sga::mbar_init(sga::smem_u32(&mma_bar), 1);
    abort_flag = 0;
    sga::fence_barrier_init();
  }
  if (warp == 0) {
    sga::tmem_alloc(sga::smem_u32(&tmem_slot), kGradTmemCols);
    sga::tmem_relinquish();
  }
  load_slot_rows(p, row, c, slot_row);
  if (t < kIdxHeads) wj[t] = bf(p.w[static_cast<size_t>(row) * kIdxHeads + t]);
  sga::tc_fence_before();
  __syncthreads();
  sga::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  {
    // q_idx and the chunk's key rows into swizzled boxes (16-byte pieces; empty slots zero-filled);
    // they land while the objective below is computed
    const uint16_t* qirow = p.q_idx + static_cast<size_t>(row) * kIdxHeads * kIdxDim;
    for (int e = t; e < kIdxHeads * 16; e += kThreads) {
      const int r = e >> 4, pc = e & 15;
      sga::cp_async_16(qi_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4), qirow + r * kIdxDim + pc * 8,
                       16);
    }
    for (int e = t; e < kChunk * 16; e += kThreads) {
      const int r = e >> 4, pc = e & 15, sr = slot_row[r];
      const uint16_t* src = p.k_idx + (seq_base + (sr >= 0 ? sr : 0)) * kIdxDim + pc * 8;
      sga::cp_async_16(ki_s + (pc >> 3) * kBox + r * 128 + (((pc & 7) ^ (r & 7)) << 4), src, sr >= 0 ? 16u : 0u);
    }
  }
  // The above reads the caller's inputs only; the statistics, z, a and the
  // scores below come from kernel A, and the gradients added into at the end
  // were cleared by the first kernel B.
  sga::grid_dependency_wait();
  sga::grid_launch_dependents();
  // ---- the target's per-head statistics: the chunks' (max, sum) pairs merged.  A query has at
  // most 32 chunks, one pair per lane; a warp loads all of its heads' pairs before reducing any.
  {
    constexpr int kHeadsPerWarp = kHeads / (kThreads / 32);
    static_assert(SGA_MAX_TOP_K / kChunk <= 32, "one chunk per lane");
    float2 v[kHeadsPerWarp];
#pragma unroll
    for (int i = 0; i < kHeadsPerWarp; ++i) {
      const int h = warp + i * (kThreads / 32);
      v[i] = lane < nch ? p.stats[(static_cast<size_t>(row) * kHeads + h) * nch + lane] : make_float2(-INFINITY, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kHeadsPerWarp; ++i) {
      const int h = warp + i * (kThreads / 32);
      const float m = warp_max(v[i].x);
      float l = 0.f;
      if (m != -INFINITY && v[i].x != -INFINITY) l = v[i].y * expf(v[i].x - m);
      l = warp_sum(l);
      if (lane == 0) {
        hm[h] = m;
        hinv[h] = l > 0.f ? 1.f / l : 0.f;
      }
    }
  }
  // ---- the indexer softmax's normaliser over the query's valid slots: the chunks' (max, sum) pairs merged
  const float* zr = p.z + static_cast<size_t>(row) * kHeads * K;
  const float* sr = p.score + static_cast<size_t>(row) * K;
  float smax = -INFINITY, ssum = 0.f;
  {
    const float2* st = p.score_stats + static_cast<size_t>(row) * nch;
    for (int cc = t; cc < nch; cc += kThreads) smax = fmaxf(smax, st[cc].x);
    smax = block_reduce<true>(smax, red);
    if (smax != -INFINITY)
      for (int cc = t; cc < nch; cc += kThreads)
        if (st[cc].x != -INFINITY) ssum += st[cc].y * expf(st[cc].x - smax);
    ssum = block_reduce<false>(ssum, red);  // (its barriers also publish hm and hinv)
  }
  // ---- p(s) for the chunk's slots: thread (slot s, head group hg) sums 16 heads
  {
    const int s = t & (kChunk - 1), hg = t / kChunk;
    constexpr int kHeadsPerGroup = kHeads / (kThreads / kChunk);
    const float* zc = zr + static_cast<size_t>(c) * kChunk + s;
    float pp = 0.f;
    if (slot_row[s] >= 0) {
      float zv[kHeadsPerGroup];  // all loads in flight at once
#pragma unroll
      for (int i = 0; i < kHeadsPerGroup; ++i) zv[i] = zc[static_cast<size_t>(hg * kHeadsPerGroup + i) * K];
#pragma unroll
      for (int i = 0; i < kHeadsPerGroup; ++i) {
        const int h = hg * kHeadsPerGroup + i;
        pp += expf(zv[i] - hm[h]) * hinv[h];
      }
    }
    pp_part[hg][s] = pp;
  }
  __syncthreads();
  float term = 0.f;
  if (t < kChunk) {
    float g = 0.f;
    if (slot_row[t] >= 0) {
      float pp = 0.f;
#pragma unroll
      for (int hg = 0; hg < kThreads / kChunk; ++hg) pp += pp_part[hg][t];
      pp *= 1.f / kHeads;
      const float log_r = sr[static_cast<size_t>(c) * kChunk + t] - smax - logf(ssum);
      if (pp > 0.f) term = pp * (logf(pp) - log_r);
      g = expf(log_r) - pp;
    }
    gs[t] = g;
  }
  term = block_reduce<false>(term, red);  // (its barriers also publish gs)
  if (t == 0) p.loss_part[static_cast<size_t>(row) * nch + c] = term;
  // ---- act (two bf16 parts) and dw: thread (j, 16 slots from s0)
  {
    const int j = t >> 2, s0 = (t & 3) * 16;
    const float4* ap = reinterpret_cast<const float4*>(
        p.a + (static_cast<size_t>(row) * kIdxHeads + j) * K + static_cast<size_t>(c) * kChunk + s0);
    float av[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = ap[i];
      av[4 * i] = v.x;
      av[4 * i + 1] = v.y;
      av[4 * i + 2] = v.z;
      av[4 * i + 3] = v.w;
    }
    float dw = 0.f;
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float x[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int s = s0 + 2 * i + e;
        const bool on = slot_row[s] >= 0 && av[2 * i + e] > 0.f;
        x[e] = on ? gs[s] * wj[j] : 0.f;
        if (on) dw = fmaf(gs[s], av[2 * i + e], dw);
      }
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(x[0], x[1]);
      hi[i] = *reinterpret_cast<const uint32_t*>(&h2);
      const float2 hf = __bfloat1622float2(h2);
      const __nv_bfloat162 l2 = __floats2bfloat162_rn(x[0] - hf.x, x[1] - hf.y);
      lo[i] = *reinterpret_cast<const uint32_t*>(&l2);
    }
    // row j of each act box: 16-byte pieces s0 / 8 and s0 / 8 + 1, swizzled
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int piece = (s0 >> 3) + q;
      const uint32_t off = j * 128 + ((piece ^ (j & 7)) << 4);
      *reinterpret_cast<uint4*>(ah_ptr + off) = make_uint4(hi[4 * q], hi[4 * q + 1], hi[4 * q + 2], hi[4 * q + 3]);
      *reinterpret_cast<uint4*>(ah_ptr + kBox + off) =
          make_uint4(lo[4 * q], lo[4 * q + 1], lo[4 * q + 2], lo[4 * q + 3]);
    }
    dw += __shfl_xor_sync(0xffffffffu, dw, 1);
    dw += __shfl_xor_sync(0xffffffffu, dw, 2);
    if ((t & 3) == 0) atomicAdd(&p.grad_w[static_cast<size_t>(row) * kIdxHeads + j], dw);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  sga::fence_proxy_async_smem();  // cp.async and st.shared writes, read by the tensor core
  __syncthreads();
  if (t == 0) {
    constexpr uint32_t idesc_dq = sga::idesc_bf16_f32(kIdxHeads, kIdxDim, false, true);
    constexpr uint32_t idesc_dk = sga::idesc_bf16_f32(kChunk, kIdxDim, true, true);
    sga::tc_fence_after();
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int part = 0; part < 2; ++part)
        sga::mma_bf16(tmem, sga::sdesc_sw128((part ? al_s : ah_s) + kk * 32, 16, 1024),
                      sga::sdesc_sw128(ki_s + kk * 2048, kBox, 1024), idesc_dq, (kk | part) ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
#pragma unroll
      for (int part = 0; part < 2; ++part)
        sga::mma_bf16(tmem + kIdxDim, sga::sdesc_sw128((part ? al_s : ah_s) + kk * 2048, kBox, 1024),
                      sga::sdesc_sw128(qi_s + kk * 2048, kBox, 1024), idesc_dk, (kk | part) ? 1u : 0u);
    sga::mma_commit(sga::smem_u32(&mma_bar));
  }
  bool ok = sga::mbar_wait(sga::smem_u32(&mma_bar), 0, &abort_flag);
  if (!ok) {
    atomicCAS(p.status, 0, static_cast<int>(SGA_ERR_TIMEOUT));
    abort_flag = 1;
  }
  ok = __syncthreads_and(ok) != 0;  // the epilogue's loads need whole warps
  sga::tc_fence_after();
  if (ok) {
    const int quarter = warp & 3, which = warp >> 2;  // 0: dq_idx, 1: dk
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + which * kIdxDim;
    const int m4 = lane & 3;
    const int rr[2] = {quarter * 16 + (lane >> 2), quarter * 16 + 8 + (lane >> 2)};
    for (int half = 0; half < 2; ++half) {
      float v[32];
      sga::tmem_ld_16x256b_x8(taddr + 64 * half, v);
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float* dst;
        if (which == 0) {
          dst = p.grad_q_idx + (static_cast<size_t>(row) * kIdxHeads + rr[i]) * kIdxDim;
        } else {
          const int r = slot_row[rr[i]];
          if (r < 0) continue;
          dst = p.grad_k_idx + (seq_base + r) * kIdxDim;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          atomicAdd(reinterpret_cast<float2*>(dst + 64 * half + 8 * k + 2 * m4),
                    make_float2(v[4 * k + 2 * i], v[4 * k + 2 * i + 1]));
      }
    }
  } else if (t == 0) {
    volatile int never = 0;
    sga::mbar_wait(sga::smem_u32(&mma_bar), 0, &never);  // its MMAs must finish before tensor memory is freed
  }
  sga::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    sga::tc_fence_after();
    sga::tmem_dealloc(tmem, kGradTmemCols);
  }
}

// B: per query, the loss (the chunks' terms summed in chunk order); also clears
// the query's q_idx and w gradients, which the next call's kernel C adds into.
__global__ void __launch_bounds__(kThreads) warmup_loss_kernel(WarmupArgs p, bool clear_grads) {
  const int row = blockIdx.x, t = threadIdx.x;
  const int nch = p.top_k / kChunk;
  // the terms come from kernel C; the gradients cleared here may still be read by earlier work
  sga::grid_dependency_wait();
  sga::grid_launch_dependents();
  if (t < 32 && !clear_grads) {
    // all of the query's terms loaded at once (at most 32 chunks, one per lane), then summed in chunk order
    const float v = t < nch ? p.loss_part[static_cast<size_t>(row) * nch + t] : 0.f;
    float sum = 0.f;
    for (int cc = 0; cc < nch; ++cc) sum += __shfl_sync(0xFFFFFFFFu, v, cc);
    if (t == 0) p.loss[row] = sum;
  }
  if (clear_grads) {
    for (int e = t; e < kIdxHeads * kIdxDim; e += kThreads)
      p.grad_q_idx[static_cast<size_t>(row) * kIdxHeads * kIdxDim + e] = 0.f;
    if (t < kIdxHeads) p.grad_w[static_cast<size_t>(row) * kIdxHeads + t] = 0.f;
  }
}

struct WarmupLayout {
  size_t z = 0, a = 0, score = 0, stats = 0, score_stats = 0, loss_part = 0, total = 0;
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
  l.stats = off;
  off += align_up(rows * kHeads * (K / kChunk) * 8);
  l.score_stats = off;
  off += align_up(rows * (K / kChunk) * 8);
  l.loss_part = off;
  off += align_up(rows * (K / kChunk) * 4);
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
      !aligned(idx, 4) || !aligned(loss, 4) || !aligned(grad_q_idx, 8) || !aligned(grad_w, 4) ||
      !aligned(grad_k_idx, 8))
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
               at<float>(ws, l.a), at<float>(ws, l.score), at<float>(ws, l.loss_part), at<float2>(ws, l.stats),
               at<float2>(ws, l.score_stats), at<int>(ws, 0), dims->n_q,
               dims->kv_stride, dims->top_k};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int rows = dims->batch * dims->n_q;
  const dim3 grid(dims->top_k / kChunk, rows);
  // Every launch is programmatic: each kernel's set-up overlaps the previous
  // kernel's tail, and its grid_dependency_wait orders what depends on it.
  cudaError_t e = launch_pdl(warmup_loss_kernel, dim3(rows), dim3(kThreads), 0, s, a, true);
  if (e == cudaSuccess) e = launch_pdl(warmup_logits_kernel, grid, dim3(kLogitThreads), kLogitsSmem, s, a);
  if (e == cudaSuccess) e = launch_pdl(warmup_grad_kernel, grid, dim3(kThreads), kGradSmem, s, a);
  if (e == cudaSuccess) e = launch_pdl(warmup_loss_kernel, dim3(rows), dim3(kThreads), 0, s, a, false);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_CUDA;
  }
  return SGA_OK;
}

}  // extern "C"
