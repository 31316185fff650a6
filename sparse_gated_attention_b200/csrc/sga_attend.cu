// Steps 3-4: sparse MLA attention in latent form over the selected positions,
// then the head-specific sigmoid output gate (archdb "A.X K2", attention
// fields: 64 heads, qk head dim 192 = 128 nope + 64 rope, KV latent 512 + rope
// 64; gate field: sigmoid gate on the attention output before o_proj).
//
// For one query: Q [64 heads x 576], rows C_s [576] for s in idx,
//   S = Q C^T * 192^-0.5,  P = softmax_s(S),  O = P C[:, 0:512],  out = O * sigmoid(g)
//
// Kernel design (one CTA per (query, split of the K selected slots)):
//   * Shared memory: Q (9 swizzled 64x64 boxes, 72 KB, loaded once by TMA), a
//     17-slot ring of 8 KB boxes holding gathered rows, and P (hi and lo bf16
//     parts, 8 KB each).
//   * Warps 0-3 gather a 64-row tile as 9 boxes [rope dims 512..575, then
//     value dims 0..63, ..., 448..511] with 16-byte cp.async copies written
//     straight into the 128-byte-swizzled layout (each warp instruction moves
//     four full 128-byte row strips; empty slots are zero-filled without a
//     read), completing on the box's mbarrier.  Warp 0 also publishes a 64-bit
//     mask of non-empty slots per tile and loads Q with TMA.
//   * Warp 4 issues tcgen05.mma: S_j = Q C_j^T (M = 64 heads, N = 64 rows,
//     K = 576) into one of two TMEM S buffers, and O += P_j V_j as 8 MMAs of
//     M = 64, N = 64 dims, K = 64 rows each, for P_hi and P_lo (P split into
//     two bf16 parts keeps ~16 mantissa bits of P).  S_{j+1} is issued before
//     PV_j so the softmax of tile j overlaps the next QK^T.
//   * Warps 5-8 (one per TMEM lane quarter, 16 heads each) run the softmax in
//     the log2 domain with a lazy running max (O in TMEM is rescaled only when
//     the max grows by more than 2^8), write P to shared memory in the
//     swizzled K-major layout, and finally scale O by sigmoid(g)/l.
//   * TMEM (512 columns): O for dims 0..255 in lanes 0-15 of each quarter and
//     dims 256..511 in lanes 16-31 (the two half-lane interleaves of the M = 64
//     accumulator layout), columns 0..255; S buffers at columns 256 and 320.
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
constexpr int kTile = 64;
constexpr int kBox = 64 * 128;  // 64 rows x 64 bf16 (128 B per row)
constexpr int kBoxesPerTile = 9;
constexpr int kRing = 17;       // >= 8 value boxes of tile j + 9 boxes of tile j+1
constexpr int kQBytes = 9 * kBox;
constexpr int kPBytes = kHeads * kTile * 2;
constexpr int kMaskRing = 4;
constexpr int kProducers = 128;  // warps 0-3
constexpr int kMmaWarp = 4;
constexpr int kThreads = 288;
constexpr int kTmemCols = 512;
constexpr int kSCol = 256;
// barriers: full[17] empty[17] q_full s_full[2] s_free[2] p_full p_free o_full mask_full[4] mask_empty[4]
constexpr int kNumBars = 2 * kRing + 1 + 2 + 2 + 3 + 2 * kMaskRing;
constexpr size_t kSmemBytes = 1024 + kRing * kBox + kQBytes + 2 * kPBytes + kNumBars * 8 + kMaskRing * 8 + 16;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kRing >= 2 * kBoxesPerTile - 1, "ring must hold a tile's values plus the next tile");

struct AttendParams {
  const uint16_t* kv;
  const int32_t* idx;
  const uint16_t* gate;
  float* out;
  float* part_o;
  float* part_ml;
  int* status;
  int n_q, kv_stride, top_k, splits, tiles_per_split;
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
  const uint32_t ring = smem_u32(smem);
  const uint32_t q_s = ring + kRing * kBox;
  const uint32_t p_hi = q_s + kQBytes;
  const uint32_t p_lo = p_hi + kPBytes;
  uint8_t* p_hi_ptr = smem + kRing * kBox + kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRing * kBox + kQBytes + 2 * kPBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kRing + s); };
  const uint32_t q_full = bar0 + 8u * (2 * kRing);
  auto s_full = [&](int b) { return bar0 + 8u * (2 * kRing + 1 + b); };
  auto s_free = [&](int b) { return bar0 + 8u * (2 * kRing + 3 + b); };
  const uint32_t p_full = bar0 + 8u * (2 * kRing + 5);
  const uint32_t p_free = bar0 + 8u * (2 * kRing + 6);
  const uint32_t o_full = bar0 + 8u * (2 * kRing + 7);
  auto mask_full = [&](int b) { return bar0 + 8u * (2 * kRing + 8 + b); };
  auto mask_empty = [&](int b) { return bar0 + 8u * (2 * kRing + 8 + kMaskRing + b); };
  uint64_t* masks = bars + kNumBars;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(masks + kMaskRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x / p.splits;
  const int split = blockIdx.x % p.splits;
  const int ntiles = p.tiles_per_split;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRing; ++s) {
      mbar_init(full(s), kProducers);  // one cp.async arrival per producer thread
      mbar_init(empty(s), 1);
    }
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), 128);
    }
    mbar_init(p_full, 128);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    for (int b = 0; b < kMaskRing; ++b) {
      mbar_init(mask_full(b), 1);
      mbar_init(mask_empty(b), 128);
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
    const int32_t* idx_row = p.idx + static_cast<size_t>(row) * p.top_k + static_cast<size_t>(split) * ntiles * kTile;
    const uint16_t* kv_b = p.kv + static_cast<size_t>(b) * p.kv_stride * kDq;
    const int ptid = threadIdx.x;
    const int part = ptid & 7;   // 16-byte chunk of a 128-byte row strip
    const int rsub = ptid >> 3;  // rows rsub + 16 i, i = 0..3
    bool ok = true;
    if (ptid == 0) {
      mbar_arrive_expect_tx(q_full, kQBytes);
      const uint64_t pol = policy_evict_first();
      for (int c = 0; c < 9; ++c) tma_load_2d(q_s + c * kBox, &qmap, q_full, c * 64, row * kHeads, pol);
    }
    for (int j = 0; j < ntiles && ok; ++j) {
      if (warp == 0) {
        const int2 v = __ldg(reinterpret_cast<const int2*>(idx_row + j * kTile) + lane);
        const bool ok0 = v.x >= 0 && v.x < p.kv_stride;
        const bool ok1 = v.y >= 0 && v.y < p.kv_stride;
        if ((v.x < -1 || v.x >= p.kv_stride) || (v.y < -1 || v.y >= p.kv_stride))
          record_status(p.status, kStatusDeviceArg);
        // 64-bit mask of filled slots: bit r <-> tile row r (lane l holds rows 2l, 2l+1)
        uint64_t m = (static_cast<uint64_t>(ok0) << (2 * lane)) | (static_cast<uint64_t>(ok1) << (2 * lane + 1));
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
      const uint16_t* src[4];
      uint32_t nbytes[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int s = __ldg(idx_row + j * kTile + rsub + 16 * i);
        const bool valid = s >= 0 && s < p.kv_stride;
        src[i] = kv_b + static_cast<size_t>(valid ? s : 0) * kDq + part * 8;
        nbytes[i] = valid ? 16u : 0u;
      }
      for (int c = 0; c < kBoxesPerTile; ++c) {
        const long long n = static_cast<long long>(j) * kBoxesPerTile + c;
        const int slot = static_cast<int>(n % kRing);
        if (!mbar_wait(empty(slot), static_cast<uint32_t>((n / kRing) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const int dim0 = c == 0 ? kDv : (c - 1) * 64;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = rsub + 16 * i;
          cp_async_16(ring + slot * kBox + r * 128 + ((part ^ (r & 7)) << 4), src[i] + dim0, nbytes[i]);
        }
        cp_async_arrive_noinc(full(slot));
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
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kHeads, kTile, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kHeads, 64, false, true);
      bool ok = mbar_wait(q_full, 0, abort_flag);
      auto issue_qk = [&](int j) -> bool {
        const int sb = j & 1;
        if (!mbar_wait(s_free(sb), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, abort_flag)) return false;
        const uint32_t d = tmem + kSCol + sb * kTile;
        int rope_slot = 0;
        for (int c = 0; c < kBoxesPerTile; ++c) {
          const long long n = static_cast<long long>(j) * kBoxesPerTile + c;
          const int slot = static_cast<int>(n % kRing);
          if (!mbar_wait(full(slot), static_cast<uint32_t>((n / kRing) & 1), abort_flag)) return false;
          fence_proxy_async_smem();  // the box was written by cp.async (generic proxy)
          tc_fence_after();
          if (c == 0) rope_slot = slot;
          const int qbox = c == 0 ? 8 : c - 1;  // Q box covering the same dims
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(d, sdesc_sw128(q_s + qbox * kBox + kk * 32, 16, 1024),
                     sdesc_sw128(ring + slot * kBox + kk * 32, 16, 1024), idesc_qk, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(s_full(sb));
        mma_commit(empty(rope_slot));  // rope dims are not needed for P V
        return true;
      };
      if (ok && ntiles > 0) ok = issue_qk(0);
      for (int j = 0; j < ntiles && ok; ++j) {
        if (j + 1 < ntiles && !(ok = issue_qk(j + 1))) break;
        if (!(ok = mbar_wait(p_full, static_cast<uint32_t>(j & 1), abort_flag))) break;
        tc_fence_after();
        for (int c = 1; c < kBoxesPerTile; ++c) {
          const long long n = static_cast<long long>(j) * kBoxesPerTile + c;
          const int slot = static_cast<int>(n % kRing);
          const int vbox = c - 1;
          const uint32_t d = vbox < 4 ? tmem + vbox * 64 : tmem + (16u << 16) + (vbox - 4) * 64;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bdesc = sdesc_sw128(ring + slot * kBox + kk * 2048, kBox, 1024);
            mma_bf16(d, sdesc_sw128(p_hi + kk * 32, 16, 1024), bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
            mma_bf16(d, sdesc_sw128(p_lo + kk * 32, 16, 1024), bdesc, idesc_pv, 1u);
          }
          mma_commit(empty(slot));
        }
        mma_commit(p_free);
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
    const int hl = lane & 15;
    const int head = quarter * 16 + hl;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (!(ok = mbar_wait(s_full(sb), static_cast<uint32_t>((j >> 1) & 1), abort_flag))) break;
      tc_fence_after();
      float s[64];
      {
        float a0[32], a1[32];
        tmem_ld32(tmem + lane_addr + kSCol + sb * kTile, a0);
        tmem_ld32(tmem + lane_addr + kSCol + sb * kTile + 32, a1);
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
      const uint64_t mask = masks[mb];
      mbar_arrive(mask_empty(mb));

      float mt = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        s[i] = ((mask >> i) & 1ull) ? s[i] * p.scale_log2 : -INFINITY;
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
      if (m_ref == -INFINITY) {
#pragma unroll
        for (int i = 0; i < 64; ++i) s[i] = 0.f;
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          s[i] = exp2f(s[i] - m_ref);
          psum += s[i];
        }
      }
      l_run = l_run * alpha + psum;

      // PV_{j-1} must be done before P and O are touched.
      if (!(ok = mbar_wait(p_free, static_cast<uint32_t>(j & 1) ^ 1u, abort_flag))) break;
      tc_fence_after();
      const bool any_resc = __any_sync(0xFFFFFFFFu, lane < 16 && resc);
      if (any_resc) {
        const float a = __shfl_sync(0xFFFFFFFFu, (lane < 16 && resc) ? alpha : 1.f, hl);
        for (int c = 0; c < 8; ++c) {
          float o[32];
          tmem_ld32(tmem + lane_addr + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] *= a;
          tmem_st32(tmem + lane_addr + c * 32, o);
        }
      }
      if (lane < 16) {
        // P[head][row] in the 128-byte-swizzled K-major layout (8 rows per 1 KB atom)
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
      const float m_h = __shfl_sync(0xFFFFFFFFu, m_ref, hl);
      const float l_h = __shfl_sync(0xFFFFFFFFu, l_run, hl);
      const int part = lane >> 4;  // 0: dims 0..255, 1: dims 256..511
      float factor = 1.f;
      float* dst;
      if (p.splits == 1) {
        const float g = p.gate ? sigmoidf_(bf16_bits_to_float(p.gate[static_cast<size_t>(row) * kHeads + head])) : 1.f;
        factor = l_h > 0.f ? g / l_h : 0.f;
        dst = p.out + (static_cast<size_t>(row) * kHeads + head) * kDv + part * 256;
      } else {
        const size_t slot = (static_cast<size_t>(row) * p.splits + split) * kHeads + head;
        dst = p.part_o + slot * kDv + part * 256;
        if (lane < 16) {
          p.part_ml[slot * 2 + 0] = m_h;
          p.part_ml[slot * 2 + 1] = l_h;
        }
      }
      for (int c = 0; c < 8; ++c) {
        float o[32];
        tmem_ld32(tmem + lane_addr + c * 32, o);
        float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          d4[i] = make_float4(o[4 * i] * factor, o[4 * i + 1] * factor, o[4 * i + 2] * factor, o[4 * i + 3] * factor);
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
  const int tiles = top_k / kTile;
  int best = 1;
  for (int s = 1; s <= tiles && s <= 64; ++s) {
    if (tiles % s == 0 && static_cast<long long>(rows) * s <= 148) best = s;
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
  p.tiles_per_split = a.top_k / kTile / splits;
  p.scale_log2 = static_cast<float>(0.07216878364870322 * 1.4426950408889634);
  sga_attend_kernel<<<rows * splits, kThreads, kSmemBytes, stream>>>(qmap, p);
  e = cudaGetLastError();
  if (e != cudaSuccess || splits == 1) return e;
  sga_combine_kernel<<<rows * kHeads, 128, 0, stream>>>(a.part_o, a.part_ml, a.gate, a.out, splits);
  return cudaGetLastError();
}

}  // namespace sga
