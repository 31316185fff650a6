// Steps 3-4: sparse MLA attention in latent form over the selected positions,
// then the head-specific sigmoid output gate (archdb "A.X K2", attention
// fields: 64 heads, qk head dim 192 = 128 nope + 64 rope, KV latent 512 + rope
// 64; gate field: sigmoid gate on the attention output before o_proj).
//
// For one query: Q [64 heads x 576], rows C_s [576] for s in idx,
//   S = Q C^T * 192^-0.5,  P = softmax_s(S),  O = P C[:, 0:512],  out = O * sigmoid(g)
//
// Kernel design (one CTA per (query, split of the K selected slots); the
// selected rows are processed in chunks of 64, each gathered exactly once):
//   * QK^T: S_j [64 heads x 64 rows] = Q C_j^T, M = 64, N = 64, K = 576, with
//     Q (72 KB, 9 swizzled boxes, TMA) in shared memory and S in TMEM (two
//     buffers).
//   * PV in transposed form: O^T [512 dims x 64 heads] += V_j^T P_j^T as four
//     M = 128 dim blocks, N = 64 heads, K = 64 rows; A = V^T read straight
//     from the gathered rows (MN-major), B = P^T from the softmax (K-major).
//     P is split into two bf16 parts (hi + lo, ~16 mantissa bits) so the
//     result keeps the accuracy of an fp32 P.  tcgen05.mma costs ~70 cycles
//     per instruction at these sizes and ~220 when consecutive MMAs change
//     accumulator, so each accumulator gets its MMAs back to back.
//   * The value dims of a chunk arrive as four 16 KB "pair" slots (two
//     swizzled 64-dim boxes each, so one M = 128 block of V^T has a fixed box
//     stride) in an 8-slot ring, i.e. two chunks; the rope dims use one 8 KB
//     slot that is freed right after QK^T.  QK^T(j+1) is issued before PV(j),
//     so the softmax of chunk j overlaps the next QK^T and chunk j+2 streams in
//     while chunk j's values wait for P.
//   * Warps 0-3 gather with 16-byte cp.async written straight into the
//     128-byte-swizzled layout (empty slots zero-filled without a read);
//     warp 0 also publishes the validity mask of each chunk and loads Q.
//     Warp 4 issues the MMAs.  Warps 5-8 (one per TMEM lane quarter, 16 heads
//     each) run the softmax in the log2 domain with a lazy running max (O is
//     rescaled only when the max grows by more than 2^8) and the epilogue.
//   * TMEM (512 columns): O^T in columns 0..255 (dim block b at 64 b, all
//     lanes), S buffers at columns 256 and 320 (M = 64 layout: lanes 0-15 of
//     each quarter).
//   * With several splits per query the CTA writes (O, m, l) partials and a
//     small combine kernel merges them and applies the gate.
#include <math.h>

#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace sga {
namespace {

constexpr int kHeads = 64;
constexpr int kDq = 576;
constexpr int kDv = 512;
constexpr int kChunk = 64;                  // selected rows per chunk
constexpr int kBoxBytes = kChunk * 128;     // 64 rows x 64 dims bf16
constexpr int kPairBytes = 2 * kBoxBytes;   // 64 rows x 128 dims
constexpr int kPairsPerChunk = 4;           // value dims 0..511
constexpr int kPairRing = 8;                // two chunks of value pairs
constexpr int kQBox = kHeads * 128;         // 64 heads x 64 dims
constexpr int kQBytes = 9 * kQBox;
constexpr int kPBytes = kHeads * kChunk * 2;  // 64 heads x 64 rows bf16
constexpr int kMaskRing = 4;
constexpr int kProducers = 128;             // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kSoftmaxThreads = 128;        // warps 5-8
constexpr int kThreads = 288;
constexpr int kTmemCols = 512;
constexpr int kSCol = 256;
// barriers: pair_full[8] pair_empty[8] rope_full rope_empty q_full s_full[2] s_free[2]
//           p_full p_free o_full mask_full[4] mask_empty[4]
constexpr int kNumBars = 2 * kPairRing + 2 + 1 + 2 + 2 + 3 + 2 * kMaskRing;
constexpr size_t kSmemBytes = 1024 + kPairRing * kPairBytes + kBoxBytes + kQBytes + 2 * kPBytes + kNumBars * 8 +
                              kMaskRing * 8 + kHeads * 4 + 16;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");

struct AttendParams {
  const uint16_t* kv;
  const int32_t* idx;
  const uint16_t* gate;
  float* out;
  float* part_o;
  float* part_ml;
  int* status;
  int n_q, kv_stride, top_k, splits, chunks_per_split;
  float scale_log2;
};

__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    sga_attend_kernel(const __grid_constant__ CUtensorMap qmap, AttendParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t pairs = smem_u32(smem);
  const uint32_t rope = pairs + kPairRing * kPairBytes;
  const uint32_t q_s = rope + kBoxBytes;
  const uint32_t p_hi = q_s + kQBytes;
  const uint32_t p_lo = p_hi + kPBytes;
  uint8_t* p_hi_ptr = smem + kPairRing * kPairBytes + kBoxBytes + kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(p_hi_ptr + 2 * kPBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto pair_full = [&](int s) { return bar0 + 8u * s; };
  auto pair_empty = [&](int s) { return bar0 + 8u * (kPairRing + s); };
  const uint32_t rope_full = bar0 + 8u * (2 * kPairRing);
  const uint32_t rope_empty = rope_full + 8u;
  const uint32_t q_full = rope_full + 16u;
  auto s_full = [&](int b) { return q_full + 8u * (1 + b); };
  auto s_free = [&](int b) { return q_full + 8u * (3 + b); };
  const uint32_t p_full = q_full + 8u * 5;
  const uint32_t p_free = q_full + 8u * 6;
  const uint32_t o_full = q_full + 8u * 7;
  auto mask_full = [&](int b) { return q_full + 8u * (8 + b); };
  auto mask_empty = [&](int b) { return q_full + 8u * (8 + kMaskRing + b); };
  uint64_t* masks = bars + kNumBars;
  float* head_f = reinterpret_cast<float*>(masks + kMaskRing);  // [64] per-head factors
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(head_f + kHeads);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int nchunks = p.chunks_per_split;
  const int slot_base = split * nchunks * kChunk;  // first selected slot of this split

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairRing; ++s) {
      mbar_init(pair_full(s), kProducers);  // one cp.async arrival per producer thread
      mbar_init(pair_empty(s), 1);
    }
    mbar_init(rope_full, kProducers);
    mbar_init(rope_empty, 1);
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), kSoftmaxThreads);
    }
    mbar_init(p_full, kSoftmaxThreads);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    for (int b = 0; b < kMaskRing; ++b) {
      mbar_init(mask_full(b), 1);
      mbar_init(mask_empty(b), kSoftmaxThreads);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&qmap);
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < kProducers / 32) {
    // ------------------------------------------------------------ gather producers
    const int b = row / p.n_q;
    const int32_t* idx_row = p.idx + static_cast<size_t>(row) * p.top_k;
    const uint16_t* kv_b = p.kv + static_cast<size_t>(b) * p.kv_stride * kDq;
    const int ptid = threadIdx.x;
    const int part = ptid & 7;   // 16-byte chunk of a 128-byte row strip
    const int rsub = ptid >> 3;  // rows rsub + 16 i, i = 0..3
    bool ok = true;
    if (ptid == 0) {
      mbar_arrive_expect_tx(q_full, kQBytes);
      const uint64_t pol = policy_evict_first();
      for (int c = 0; c < 9; ++c) tma_load_2d(q_s + c * kQBox, &qmap, q_full, c * 64, row * kHeads, pol);
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      const int first = slot_base + j * kChunk;
      if (warp == 0) {
        // validity mask of this chunk's 64 slots (bit r <-> chunk row r)
        bool v0 = false, v1 = false;
        const int r0 = first + 2 * lane;
        if (r0 < p.top_k) {
          const int2 v = __ldg(reinterpret_cast<const int2*>(idx_row + r0));
          v0 = v.x >= 0 && v.x < p.kv_stride;
          v1 = v.y >= 0 && v.y < p.kv_stride;
          if (v.x < -1 || v.x >= p.kv_stride || v.y < -1 || v.y >= p.kv_stride)
            record_status(p.status, kStatusDeviceArg);
        }
        uint64_t m = (static_cast<uint64_t>(v0) << (2 * lane)) | (static_cast<uint64_t>(v1) << (2 * lane + 1));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m |= __shfl_xor_sync(0xFFFFFFFFu, m, o);
        if (lane == 0) {
          const int mb = j % kMaskRing;
          if (mbar_wait(mask_empty(mb), static_cast<uint32_t>((j / kMaskRing) & 1) ^ 1u, abort_flag)) {
            masks[mb] = m;
            mbar_arrive(mask_full(mb));
          } else {
            ok = false;
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      // this thread's four rows of the chunk
      const uint16_t* src[4];
      uint32_t nbytes[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int sidx = first + rsub + 16 * i;
        int s = -1;
        if (sidx < p.top_k) s = __ldg(idx_row + sidx);
        const bool valid = s >= 0 && s < p.kv_stride;
        src[i] = kv_b + static_cast<size_t>(valid ? s : 0) * kDq + part * 8;
        nbytes[i] = valid ? 16u : 0u;
      }
      // rope dims 512..575 -> the rope slot
      if (!mbar_wait(rope_empty, static_cast<uint32_t>(j & 1) ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = rsub + 16 * i;
        cp_async_16(rope + r * 128 + ((part ^ (r & 7)) << 4), src[i] + kDv, nbytes[i]);
      }
      cp_async_arrive_noinc(rope_full);
      // value dims 128 q .. 128 q + 127 -> pair slot (4 j + q) mod 8
      for (int q = 0; q < kPairsPerChunk; ++q) {
        const int n = j * kPairsPerChunk + q;
        const int slot = n % kPairRing;
        if (!mbar_wait(pair_empty(slot), static_cast<uint32_t>((n / kPairRing) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t base = pairs + slot * kPairBytes;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rsub + 16 * i;
          const uint32_t dst = base + r * 128 + ((part ^ (r & 7)) << 4);
          cp_async_16(dst, src[i] + 128 * q, nbytes[i]);
          cp_async_16(dst + kBoxBytes, src[i] + 128 * q + 64, nbytes[i]);
        }
        cp_async_arrive_noinc(pair_full(slot));
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      *abort_flag = 1;
      if (ptid == 0) {
        volatile int never = 0;
        mbar_wait(q_full, 0, &never);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kHeads, kChunk, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kHeads, true, false);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      auto wait_full = [&](uint32_t bar, uint32_t parity) -> bool {
        if (!mbar_wait(bar, parity, abort_flag)) return false;
        fence_proxy_async_smem();  // written by cp.async (generic proxy)
        tc_fence_after();
        return true;
      };
      auto issue_qk = [&](int j) -> bool {
        const int sb = j & 1;
        if (!mbar_wait(s_free(sb), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + sb * kChunk;
        if (!wait_full(rope_full, static_cast<uint32_t>(j & 1))) return false;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_bf16(d, sdesc_sw128(q_s + 8 * kQBox + kk * 32, 16, 1024), sdesc_sw128(rope + kk * 32, 16, 1024),
                   idesc_qk, kk > 0 ? 1u : 0u);
        mma_commit(rope_empty);  // rope dims are not needed for P V
        for (int q = 0; q < kPairsPerChunk; ++q) {
          const int n = j * kPairsPerChunk + q;
          const int slot = n % kPairRing;
          if (!wait_full(pair_full(slot), static_cast<uint32_t>((n / kPairRing) & 1))) return false;
          const uint32_t base = pairs + slot * kPairBytes;
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d, sdesc_sw128(q_s + (2 * q + bx) * kQBox + kk * 32, 16, 1024),
                       sdesc_sw128(base + bx * kBoxBytes + kk * 32, 16, 1024), idesc_qk, 1u);
          }
        }
        mma_commit(s_full(sb));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        if (!mbar_wait(p_full, static_cast<uint32_t>(j & 1), abort_flag)) return false;
        tc_fence_after();
        for (int q = 0; q < kPairsPerChunk; ++q) {
          const int slot = (j * kPairsPerChunk + q) % kPairRing;
          const uint32_t base = pairs + slot * kPairBytes;
          const uint32_t d = tmem + q * kHeads;  // O^T block: dims 128 q .. +127
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // A = V^T: M = 128 dims over the pair's two boxes, K = rows 16 kk ..
            const uint64_t adesc = sdesc_sw128(base + kk * 2048, kBoxBytes, 1024);
#pragma unroll
            for (int part = 0; part < 2; ++part) {
              const uint64_t bdesc = sdesc_sw128((part ? p_lo : p_hi) + kk * 32, 16, 1024);
              mma_bf16(d, adesc, bdesc, idesc_pv, (j > 0 || kk > 0 || part > 0) ? 1u : 0u);
            }
          }
          mma_commit(pair_empty(slot));
        }
        mma_commit(p_free);
        return true;
      };
      if (ok && nchunks > 0) ok = issue_qk(0);
      for (int j = 0; j < nchunks && ok; ++j) {
        if (j + 1 < nchunks && !(ok = issue_qk(j + 1))) break;
        ok = issue_pv(j);
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(o_full);
      if (!ok) {
        volatile int never = 0;
        mbar_wait(o_full, 0, &never);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int head = quarter * 16 + (lane & 15);  // lanes 0-15 own this head's S row
    const bool owner = lane < 16;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int sb = j & 1;
      if (!(ok = mbar_wait(s_full(sb), static_cast<uint32_t>((j >> 1) & 1), abort_flag))) break;
      tc_fence_after();
      float s[64];
      {
        float a0[32], a1[32];
        tmem_ld32(tmem + lane_addr + kSCol + sb * kChunk, a0);
        tmem_ld32(tmem + lane_addr + kSCol + sb * kChunk + 32, a1);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = a0[i];
          s[32 + i] = a1[i];
        }
      }
      tc_fence_before();
      mbar_arrive(s_free(sb));
      const int mb = j % kMaskRing;
      if (!(ok = mbar_wait(mask_full(mb), static_cast<uint32_t>((j / kMaskRing) & 1), abort_flag))) break;
      const uint64_t mk = masks[mb];
      mbar_arrive(mask_empty(mb));
      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = ((mk >> i) & 1ull) ? s[i] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[i]);
      }
      float alpha = 1.f;
      bool resc = false;
      if (m_ref == -INFINITY) {
        m_ref = mt;  // nothing accumulated yet (all earlier weights were zero)
      } else if (mt > m_ref + kRescaleThreshold) {
        alpha = exp2f(m_ref - mt);
        m_ref = mt;
        resc = true;
      }
      float psum = 0.f;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = m_ref == -INFINITY ? 0.f : exp2f(s[i] - m_ref);
        psum += s[i];
      }
      l_run = l_run * alpha + psum;
      // PV_{j-1} must be done before P and O are touched.
      if (!(ok = mbar_wait(p_free, static_cast<uint32_t>(j & 1) ^ 1u, abort_flag))) break;
      tc_fence_after();
      if (owner) head_f[head] = alpha;
      if (named_barrier_or(1, kSoftmaxThreads, owner && resc)) {
        // O^T[dim][head] *= alpha[head]: every lane holds one dim of each block
        for (int blk = 0; blk < 4; ++blk) {
          for (int c = 0; c < 2; ++c) {
            float o[32];
            tmem_ld32(tmem + lane_addr + blk * kHeads + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= head_f[c * 32 + i];
            tmem_st32(tmem + lane_addr + blk * kHeads + c * 32, o);
          }
        }
        named_barrier(1, kSoftmaxThreads);
      }
      if (owner) {
        // P[head][row] in the 128-byte-swizzled K-major layout (8 heads per 1 KB atom)
        const uint32_t rbase = (head >> 3) * 1024 + (head & 7) * 128;
#pragma unroll
        for (int c8 = 0; c8 < 8; ++c8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = s[8 * c8 + 2 * e], x1 = s[8 * c8 + 2 * e + 1];
            hi[e] = pack_bf16(x0, x1);
            const float h0 = __uint_as_float(hi[e] << 16), h1 = __uint_as_float(hi[e] & 0xFFFF0000u);
            lo[e] = pack_bf16(x0 - h0, x1 - h1);
          }
          const uint32_t off = rbase + ((c8 ^ (head & 7)) << 4);
          *reinterpret_cast<uint4*>(p_hi_ptr + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(p_hi_ptr + kPBytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (!ok) {
      record_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    } else if (mbar_wait(o_full, 0, abort_flag)) {
      tc_fence_after();
      // per-head factor: gate / l (one split) or 1 (partials)
      const size_t pslot = (static_cast<size_t>(row) * p.splits + split) * kHeads;
      if (owner) {
        float f = 1.f;
        if (p.splits == 1) {
          const float g =
              p.gate ? sigmoidf_(bf16_bits_to_float(p.gate[static_cast<size_t>(row) * kHeads + head])) : 1.f;
          f = l_run > 0.f ? g / l_run : 0.f;
        } else {
          p.part_ml[(pslot + head) * 2 + 0] = m_ref;
          p.part_ml[(pslot + head) * 2 + 1] = l_run;
        }
        head_f[head] = f;
      }
      named_barrier(1, kSoftmaxThreads);
      // O^T block b: this lane holds dim 128 b + 32 quarter + lane for all 64 heads
      float* base = p.splits == 1 ? p.out + static_cast<size_t>(row) * kHeads * kDv : p.part_o + pslot * kDv;
      for (int blk = 0; blk < 4; ++blk) {
        const int dim = 128 * blk + 32 * quarter + lane;
        for (int c = 0; c < 2; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_addr + blk * kHeads + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int h = c * 32 + i;
            base[static_cast<size_t>(h) * kDv + dim] = o[i] * head_f[h];
          }
        }
      }
    } else {
      record_status(p.status, kStatusTimeout);
      *abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// Merges split partials: o = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, times sigmoid(g).
__global__ void __launch_bounds__(128) sga_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_ml,
                                                          const uint16_t* __restrict__ gate, float* __restrict__ out,
                                                          int splits) {
  const int row = blockIdx.x / kHeads;
  const int head = blockIdx.x % kHeads;
  __shared__ float wts[64];
  if (threadIdx.x < 32) {
    float mx = -INFINITY;
    for (int s = threadIdx.x; s < splits; s += 32)
      mx = fmaxf(mx, part_ml[((static_cast<size_t>(row) * splits + s) * kHeads + head) * 2]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    float lsum = 0.f;
    for (int s = threadIdx.x; s < splits; s += 32) {
      const size_t k = ((static_cast<size_t>(row) * splits + s) * kHeads + head) * 2;
      const float ms = part_ml[k];
      const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - mx);
      wts[s] = w;
      lsum += w * part_ml[k + 1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xFFFFFFFFu, lsum, o);
    const float g = gate ? sigmoidf_(bf16_bits_to_float(gate[static_cast<size_t>(row) * kHeads + head])) : 1.f;
    const float f = lsum > 0.f ? g / lsum : 0.f;
    __syncwarp();
    for (int s = threadIdx.x; s < splits; s += 32) wts[s] *= f;
  }
  __syncthreads();
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const float w = wts[s];
    const float4 v = __ldg(reinterpret_cast<const float4*>(
                               part_o + ((static_cast<size_t>(row) * splits + s) * kHeads + head) * kDv) +
                           threadIdx.x);
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  }
  reinterpret_cast<float4*>(out + (static_cast<size_t>(row) * kHeads + head) * kDv)[threadIdx.x] = acc;
}

}  // namespace

// Splits of the K slots per query so that rows * splits fills ~148 SMs once.
int attend_splits(int rows, int top_k) {
  const int chunks = (top_k + kChunk - 1) / kChunk;
  int best = 1;
  for (int s = 1; s <= chunks && s <= 64; ++s) {
    if (chunks % s == 0 && static_cast<long long>(rows) * s <= 148) best = s;
  }
  return best;
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t stream) {
  const int rows = a.batch * a.n_q;
  if (rows == 0) return cudaSuccess;
  const int splits = attend_splits(rows, a.top_k);
  CUtensorMap qmap;
  cudaError_t e = make_tmap_bf16_2d(&qmap, a.q, kDq, static_cast<uint64_t>(rows) * kHeads, kDq * 2, 64, kHeads);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(sga_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  AttendParams p;
  p.kv = a.kv;
  p.idx = a.idx;
  p.gate = a.gate;
  p.out = a.out;
  p.part_o = a.part_o;
  p.part_ml = a.part_ml;
  p.status = a.status;
  p.n_q = a.n_q;
  p.kv_stride = a.kv_stride;
  p.top_k = a.top_k;
  p.splits = splits;
  p.chunks_per_split = (a.top_k + kChunk - 1) / kChunk / splits;
  p.scale_log2 = static_cast<float>(0.07216878364870322 * 1.4426950408889634);
  sga_attend_kernel<<<rows * splits, kThreads, kSmemBytes, stream>>>(qmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  sga_combine_kernel<<<rows * kHeads, 128, 0, stream>>>(a.part_o, a.part_ml, a.gate, a.out, splits);
  return cudaGetLastError();
}

}  // namespace sga
