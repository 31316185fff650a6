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
//     result keeps the accuracy of an fp32 P.  Back-to-back tcgen05.mma
//     into one accumulator costs ~44 cycles at M = 64, N = 64 and ~48 at
//     M = 128, N = 64 (measured), so the 36 QK^T and 32 PV instructions of a
//     chunk take ~3,100 cycles of tensor time, below the chunk's gather time.
//   * The value dims of a chunk arrive as four 16 KB "pair" slots (two
//     swizzled 64-dim boxes each, so one M = 128 block of V^T has a fixed box
//     stride) in an 8-slot ring, i.e. two chunks; the rope dims use one 8 KB
//     slot that is freed right after QK^T.  QK^T(j+1) is issued before PV(j),
//     so the softmax of chunk j overlaps the next QK^T and chunk j+2 streams in
//     while chunk j's values wait for P.
//   * Warps 0-3 gather each chunk through both of the SM's copy paths at
//     once: value pairs 1-3 with TMA tile::gather4 (four cache rows x one
//     64-dim box per instruction, written by the TMA straight into the
//     128-byte-swizzled layout; each warp takes 16 rows), the rope box and
//     value pair 0 with 16-byte cp.async from all 128 threads (swizzled by
//     hand, empty slots zero-filled without a read).  An empty slot in a
//     gather4 quad gathers the sequence's row 0 and is masked out of the
//     softmax.  Warp 0 also publishes the validity mask of each chunk and
//     loads Q.
//     Warp 4 issues QK^T, polling its barriers so it never waits on one
//     operand while another is ready.  Warps 5-8 (one per TMEM lane quarter,
//     16 heads each) run the softmax in the log2 domain with a lazy running
//     max (O is rescaled only when the max grows by more than 2^8); once P_j
//     is written, one of their threads issues PV(j) itself, so value slots
//     are released (and refilled) without a round trip through the MMA warp.
//   * TMEM (512 columns): O^T in columns 0..255 (dim block b at 64 b, all
//     lanes), S buffers at columns 256 and 320 (M = 64 layout: lanes 0-15 of
//     each quarter).
//   * The splits of one query form a thread-block cluster.  Each CTA keeps its
//     (m, l) per head in shared memory; after a cluster barrier every CTA
//     reads all of them and scales its own O by 2^(m_r - M) g / L while
//     reading it out of TMEM.  CTA r owns dims [512 r / S, 512 (r+1) / S):
//     every CTA pushes its scaled O for those dims into the owner's (now
//     idle) value ring with remote shared-memory stores; after a second
//     barrier each owner sums its S buffers locally and writes them.  No
//     partials leave the chip.
#include <cooperative_groups.h>
#include <math.h>

#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace cg = cooperative_groups;

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
constexpr int kProducerWarps = 4;          // warps 0-3
constexpr int kProducers = 32 * kProducerWarps;
constexpr int kMmaWarp = 4;
constexpr int kSoftmaxThreads = 128;        // warps 5-8
constexpr int kPvThread = (4 + 1) * 32;     // the softmax thread that issues PV
constexpr int kThreads = 288;
constexpr int kTmemCols = 512;
constexpr int kSCol = 256;
// barriers: pair_full[8] pair_empty[8] rope_full rope_empty q_full s_full[2] s_free[2]
//           qk_done p_free o_full mask_full[4] mask_empty[4]
constexpr int kNumBars = 2 * kPairRing + 2 + 1 + 2 + 2 + 3 + 2 * kMaskRing;
constexpr int kMaxSplits = 8;               // splits of a query = CTAs of its cluster
constexpr size_t kSmemBytes = 1024 + kPairRing * kPairBytes + kBoxBytes + kQBytes + 2 * kPBytes + kNumBars * 8 +
                              kMaskRing * 8 + kHeads * 4 + kHeads * 8 + 16;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

static_assert(kSmemBytes <= 232448, "shared memory budget");
// the split merge's receive buffer ([S][64][4 ceil(128 / S)] fp32, at most 136 KB for S <= 8, largest at
// S = 7) lies over the value ring, the rope slot and the Q buffer, which are contiguous and idle once every
// MMA has finished
static_assert(kPairRing * kPairBytes + kBoxBytes + kQBytes >= 7 * kHeads * 76 * 4, "split merge receive buffer");

struct AttendParams {
  const uint16_t* kv;
  const int32_t* idx;
  const uint16_t* gate;
  float* out;
  uint16_t* out_bf16;  // or null
  int* status;
  int n_q, kv_stride, top_k, splits, chunks_per_split;
  float scale_log2;
};

__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + expf(-g)); }

// 2^x with the hardware approximation (relative error ~2^-22; results below
// 2^-126 flush to zero, which only drops weights far below the fp32 sum).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1)
    sga_attend_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kvmap,
                      AttendParams p) {
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
  const uint32_t qk_done = q_full + 8u * 5;  // every QK^T MMA of the MMA warp has finished
  const uint32_t p_free = q_full + 8u * 6;
  const uint32_t o_full = q_full + 8u * 7;
  auto mask_full = [&](int b) { return q_full + 8u * (8 + b); };
  auto mask_empty = [&](int b) { return q_full + 8u * (8 + kMaskRing + b); };
  uint64_t* masks = bars + kNumBars;
  float* head_f = reinterpret_cast<float*>(masks + kMaskRing);  // [64] per-head factors
  float2* own_ml = reinterpret_cast<float2*>(head_f + kHeads);   // [64] (m, l) of this split, read by the cluster
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(own_ml + kHeads);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  cg::cluster_group cluster = cg::this_cluster();
  const int row = blockIdx.x / p.splits;
  const int split = static_cast<int>(cluster.block_rank());  // the cluster is the query's p.splits CTAs
  const int nchunks = p.chunks_per_split;
  const int slot_base = split * nchunks * kChunk;  // first selected slot of this split

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairRing; ++s) {
      // pair 0 of a chunk (slots 0 and 4) arrives by cp.async from every producer
      // thread; pairs 1-3 by one gather4 expect_tx per producer warp
      mbar_init(pair_full(s), s % kPairsPerChunk == 0 ? kProducers : kProducerWarps);
      mbar_init(pair_empty(s), 1);
    }
    mbar_init(rope_full, kProducers);
    mbar_init(rope_empty, 1);
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_free(b), kSoftmaxThreads);
    }
    mbar_init(qk_done, 1);
    mbar_init(p_free, 1);
    mbar_init(o_full, 1);
    for (int b = 0; b < kMaskRing; ++b) {
      mbar_init(mask_full(b), 1);
      mbar_init(mask_empty(b), kSoftmaxThreads);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&kvmap);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Set-up above overlaps the previous kernel on the stream; indices (and
  // every input) are read below.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp < kProducerWarps) {
    // ------------------------------------------------------------ gather producers
    const int b = row / p.n_q;
    const int32_t* idx_row = p.idx + static_cast<size_t>(row) * p.top_k;
    const int row0 = b * p.kv_stride;  // this sequence's first row in the [B * L] cache map
    const int ptid = threadIdx.x;
    const int g = lane & 3;             // this lane's group of 4 rows within the warp's 16
    const int grow = 16 * warp + 4 * g;  // first chunk row of that group
    const int part = ptid & 7;          // cp.async: 16-byte piece of a 128-byte row strip
    const int rsub = ptid >> 3;         // cp.async: rows rsub + 16 i, i = 0..3
    const uint16_t* kv_b = p.kv + static_cast<size_t>(b) * p.kv_stride * kDq;
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
      // gather4: cache rows of this lane's quad (empty or invalid slots -> row 0, masked above)
      int y[4];
      {
        const int sidx = first + grow;  // a multiple of 4: one 16-byte load
        int4 v = make_int4(-1, -1, -1, -1);
        if (sidx < p.top_k) v = __ldg(reinterpret_cast<const int4*>(idx_row + sidx));
        const int e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          y[i] = row0 + ((e[i] >= 0 && e[i] < p.kv_stride) ? e[i] : 0);
          SGA_DCHECK(p.status, y[i] >= row0 && y[i] < row0 + p.kv_stride);
        }
      }
      // cp.async: this thread's four rows of the chunk (empty slots zero-filled)
      const uint16_t* src[4];
      uint32_t nbytes[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int sidx = first + rsub + 16 * i;
        int sv = -1;
        if (sidx < p.top_k) sv = __ldg(idx_row + sidx);
        const bool valid = sv >= 0 && sv < p.kv_stride;
        src[i] = kv_b + static_cast<size_t>(valid ? sv : 0) * kDq + part * 8;
        nbytes[i] = valid ? 16u : 0u;
      }
      // rope dims 512..575 -> the rope slot (cp.async)
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
        if (q == 0) {  // cp.async from every producer thread
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = rsub + 16 * i;
            const uint32_t dst = base + r * 128 + ((part ^ (r & 7)) << 4);
            cp_async_16(dst, src[i], nbytes[i]);
            cp_async_16(dst + kBoxBytes, src[i] + 64, nbytes[i]);
          }
          cp_async_arrive_noinc(pair_full(slot));
        } else {  // gather4 (lanes 0-7: quad x box)
          if (lane == 0) mbar_arrive_expect_tx(pair_full(slot), 16 * 2 * 128);
          __syncwarp();
          if (lane < 8) {
            const int bx = lane >> 2;
            tma_gather4(base + bx * kBoxBytes + grow * 128, &kvmap, pair_full(slot), 128 * q + 64 * bx, y[0], y[1],
                        y[2], y[3]);
          }
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    // On a timeout the waits above have run for about a second, long after any
    // gather issued before them has landed.
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
      bool ok = mbar_wait(q_full, 0, abort_flag);
      // Non-blocking issue of QK^T(qk_j), piece by piece: part 0 is the rope
      // box (once the S buffer and the rope slot are ready), parts 1-4 one
      // value pair each.
      int qk_j = 0, qk_part = 0;
      long long idle_since = clock64();
      while (ok && qk_j < nchunks) {
        bool did = false;
        const int sb = qk_j & 1;
        const uint32_t d = tmem + kSCol + sb * kChunk;
        if (qk_part == 0) {
          if (mbar_test_wait(s_free(sb), static_cast<uint32_t>((qk_j >> 1) & 1) ^ 1u) &&
              mbar_test_wait(rope_full, static_cast<uint32_t>(qk_j & 1))) {
            fence_proxy_async_smem();  // written by cp.async (generic proxy)
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16(d, sdesc_sw128(q_s + 8 * kQBox + kk * 32, 16, 1024), sdesc_sw128(rope + kk * 32, 16, 1024),
                       idesc_qk, kk > 0 ? 1u : 0u);
            mma_commit(rope_empty);  // rope dims are not needed for P V
            qk_part = 1;
            did = true;
          }
        } else {
          const int q = qk_part - 1;
          const int n = qk_j * kPairsPerChunk + q;
          const int slot = n % kPairRing;
          if (mbar_test_wait(pair_full(slot), static_cast<uint32_t>((n / kPairRing) & 1))) {
            fence_proxy_async_smem();
            tc_fence_after();
            const uint32_t base = pairs + slot * kPairBytes;
#pragma unroll
            for (int bx = 0; bx < 2; ++bx) {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16(d, sdesc_sw128(q_s + (2 * q + bx) * kQBox + kk * 32, 16, 1024),
                         sdesc_sw128(base + bx * kBoxBytes + kk * 32, 16, 1024), idesc_qk, 1u);
            }
            if (qk_part == kPairsPerChunk) {
              mma_commit(s_full(sb));
              ++qk_j;
              qk_part = 0;
            } else {
              ++qk_part;
            }
            did = true;
          }
        }
        if (did) {
          idle_since = clock64();
        } else if (*abort_flag || clock64() - idle_since > kWaitBudgetCycles) {
          ok = false;
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(qk_done);
      volatile int never = 0;
      mbar_wait(qk_done, 0, &never);  // every MMA this thread issued has finished
    }
  } else {
    // ------------------------------------------------------------ softmax
    // S is read with the 16-lane x 256-bit TMEM shape, which matches the M = 64
    // accumulator (16 rows per lane quarter): thread t of the warp holds rows
    // t/4 and 8 + t/4 of its quarter, columns 8k + 2(t%4) and 8k + 2(t%4) + 1
    // for k = 0..7.  The four threads of a row combine its max and sum with two
    // shuffles, so every lane works on 32 scores per chunk.
    const int quarter = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int m4 = lane & 3;
    const int hrow[2] = {quarter * 16 + (lane >> 2), quarter * 16 + 8 + (lane >> 2)};  // this thread's two heads
    float m_ref[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    // Every softmax thread runs every iteration, even after a wait ran out
    // (the abort flag then makes each later wait return at once), so the
    // named barriers below always see all 128 threads.
    bool ok = true;
    for (int j = 0; j < nchunks; ++j) {
      const int sb = j & 1;
      ok = ok && mbar_wait(s_full(sb), static_cast<uint32_t>((j >> 1) & 1), abort_flag);
      tc_fence_after();
      float r[32];
      tmem_ld_16x256b_x8(tmem + lane_addr + kSCol + sb * kChunk, r);
      tc_fence_before();
      mbar_arrive(s_free(sb));
      const int mb = j % kMaskRing;
      ok = ok && mbar_wait(mask_full(mb), static_cast<uint32_t>((j / kMaskRing) & 1), abort_flag);
      const uint64_t mk = masks[mb];
      mbar_arrive(mask_empty(mb));
      // x[i][2k + e] = score of row i at column 8k + 2 m4 + e (masked slots -> -inf)
      float x[2][16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const bool valid = (mk >> (8 * k + 2 * m4 + e)) & 1ull;
          x[0][2 * k + e] = valid ? r[4 * k + e] * p.scale_log2 : -INFINITY;
          x[1][2 * k + e] = valid ? r[4 * k + 2 + e] * p.scale_log2 : -INFINITY;
        }
      }
      float alpha[2];
      bool resc = false;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        float mp[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) mp[c] = fmaxf(fmaxf(x[i][4 * c], x[i][4 * c + 1]), fmaxf(x[i][4 * c + 2], x[i][4 * c + 3]));
        float mt = fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3]));
        mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 1));
        mt = fmaxf(mt, __shfl_xor_sync(0xFFFFFFFFu, mt, 2));
        alpha[i] = 1.f;
        if (m_ref[i] == -INFINITY) {
          m_ref[i] = mt;  // nothing accumulated yet (all earlier weights were zero)
        } else if (mt > m_ref[i] + kRescaleThreshold) {
          alpha[i] = exp2f(m_ref[i] - mt);
          m_ref[i] = mt;
          resc = true;
        }
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        if (m_ref[i] == -INFINITY) {  // every slot so far is empty: all weights are zero
#pragma unroll
          for (int c = 0; c < 16; ++c) x[i][c] = 0.f;
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            x[i][c] = fast_exp2(x[i][c] - m_ref[i]);
            ps[c & 3] += x[i][c];
          }
        }
        float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
        psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 1);
        psum += __shfl_xor_sync(0xFFFFFFFFu, psum, 2);
        l_run[i] = l_run[i] * alpha[i] + psum;
      }
      // PV_{j-1} must be done before P and O are touched.
      ok = ok && mbar_wait(p_free, static_cast<uint32_t>(j & 1) ^ 1u, abort_flag);
      tc_fence_after();
      if (m4 == 0) {
        head_f[hrow[0]] = alpha[0];
        head_f[hrow[1]] = alpha[1];
      }
      if (named_barrier_or(1, kSoftmaxThreads, resc)) {
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
      // P[head][row] in the 128-byte-swizzled K-major layout (8 heads per 1 KB
      // atom); this thread writes the bf16 pairs of columns 8k + 2 m4, +1.
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int h = hrow[i];
        const uint32_t rbase = (h >> 3) * 1024 + (h & 7) * 128 + 4 * m4;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float x0 = x[i][2 * k], x1 = x[i][2 * k + 1];
          const uint32_t hi = pack_bf16(x0, x1);
          const float h0 = __uint_as_float(hi << 16), h1 = __uint_as_float(hi & 0xFFFF0000u);
          const uint32_t lo = pack_bf16(x0 - h0, x1 - h1);
          const uint32_t off = rbase + ((k ^ (h & 7)) << 4);
          *reinterpret_cast<uint32_t*>(p_hi_ptr + off) = hi;
          *reinterpret_cast<uint32_t*>(p_hi_ptr + kPBytes + off) = lo;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_barrier(2, kSoftmaxThreads);  // P_j (and any rescale of O) complete
      if (threadIdx.x == kPvThread) {
        // PV(j): O^T[dims 128 q ..][heads] += V_j^T (P_hi + P_lo)^T, one accumulator block per value pair
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kHeads, true, false);
        tc_fence_after();
        for (int q = 0; q < kPairsPerChunk; ++q) {
          const int slot = (j * kPairsPerChunk + q) % kPairRing;
          const uint32_t base = pairs + slot * kPairBytes;
          const uint32_t d = tmem + q * kHeads;
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
      }
    }
    if (threadIdx.x == kPvThread) mma_commit(o_full);  // every PV this thread issued
    const bool have_o = ok && mbar_wait(o_full, 0, abort_flag);
    if (!have_o) {
      record_status(p.status, kStatusTimeout);
      *abort_flag = 1;
      if (threadIdx.x == kPvThread) {  // its MMAs must be done before TMEM is freed
        volatile int never = 0;
        mbar_wait(o_full, 0, &never);
      }
    }
    if (m4 == 0) {
      own_ml[hrow[0]] = make_float2(m_ref[0], l_run[0]);
      own_ml[hrow[1]] = make_float2(m_ref[1], l_run[1]);
    }
  }

  // ---- split merge: out = g / L * sum_r 2^(m_r - M) O_r with M = max_r m_r and
  // L = sum_r 2^(m_r - M) l_r (per head).  Every thread of the cluster takes
  // part in its barriers, on every path.
  const int S = p.splits;
  float* o_stage = reinterpret_cast<float*>(smem);  // value ring + rope slot + Q buffer, idle after the MMAs
  if (S > 1) {
    cluster.sync();  // every split's (m, l) published; all MMAs of every CTA done
  } else {
    __syncthreads();
  }
  if (warp > kMmaWarp && lane < 16) {
    const int head = (warp & 3) * 16 + lane;
    const float g = p.gate ? sigmoidf_(bf16_bits_to_float(p.gate[static_cast<size_t>(row) * kHeads + head])) : 1.f;
    float f;
    if (S == 1) {
      const float l = own_ml[head].y;
      f = l > 0.f ? g / l : 0.f;
    } else {
      // every split's (m, l) for this head, all loads in flight at once
      float2 ml[kMaxSplits];
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        ml[r] = r < S ? *cluster.map_shared_rank(&own_ml[head], r) : make_float2(-INFINITY, 0.f);
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r) mx = fmaxf(mx, ml[r].x);
      float L = 0.f;
#pragma unroll
      for (int r = 0; r < kMaxSplits; ++r)
        if (ml[r].x != -INFINITY) L += exp2f(ml[r].x - mx) * ml[r].y;
      const float m_own = own_ml[head].x;
      f = (L > 0.f && m_own != -INFINITY) ? exp2f(m_own - mx) * g / L : 0.f;
    }
    head_f[head] = f;
  }
  __syncthreads();
  // With several splits, CTA r owns the float4 columns [v0(r), v0(r+1)) of
  // every head's 512 dims, v0(r) = 128 r / S.  Every CTA pushes its scaled O
  // for those dims into the owner's receive buffer with remote stores (a
  // warp writes 32 consecutive dims of one head: one 128-byte line per
  // store), laid out [source split][head][kStride] fp32 over the owner's idle
  // value ring, rope slot and Q buffer; after one cluster barrier each owner
  // sums its S buffers locally.  No CTA reads another's shared memory after
  // that barrier.
  const int kStride = 4 * ((kDv / 4 + S - 1) / S);  // floats per (source, head) row: the widest slice
  float* recv = o_stage;
  if (warp < kProducerWarps || warp > kMmaWarp) {
    // Eight warps read O^T out of TMEM: warp w reads lane quarter w % 4; the
    // producer warps take dim blocks 0-1, the softmax warps blocks 2-3.
    // O^T block b: this lane holds dim 128 b + 32 quarter + lane for all 64 heads.
    const int quarter = warp & 3;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const int blk0 = warp < kProducerWarps ? 0 : 2;
    tc_fence_after();
    for (int c = 0; c < 2; ++c) {
      float hf[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) hf[i] = head_f[c * 32 + i];
      for (int blk = blk0; blk < blk0 + 2; ++blk) {
        const int dim = 128 * blk + 32 * quarter + lane;
        float o[32];
        tmem_ld32(tmem + lane_addr + blk * kHeads + c * 32, o);
        float* col;
        if (S == 1) {
          const size_t off = static_cast<size_t>(row) * kHeads * kDv + static_cast<size_t>(c * 32) * kDv + dim;
          col = p.out + off;
#pragma unroll
          for (int i = 0; i < 32; ++i) col[static_cast<size_t>(i) * kDv] = o[i] * hf[i];
          if (p.out_bf16 != nullptr) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              p.out_bf16[off + static_cast<size_t>(i) * kDv] = __bfloat16_as_ushort(__float2bfloat16_rn(o[i] * hf[i]));
          }
        } else {
          const int v = dim >> 2;
          const int owner = ((v + 1) * S - 1) / (kDv / 4);  // the r with v0(r) <= v < v0(r + 1)
          const int dl = dim - 4 * ((kDv / 4) * owner / S);
          col = cluster.map_shared_rank(recv + (split * kHeads + c * 32) * kStride + dl, owner);
#pragma unroll
          for (int i = 0; i < 32; ++i) col[i * kStride] = o[i] * hf[i];
        }
      }
    }
  }
  if (S > 1) {
    cluster.sync();  // every split's scaled O delivered to its owners
    const int v0 = (kDv / 4) * split / S, v1 = (kDv / 4) * (split + 1) / S;
    const int vecs = v1 - v0;
    float* orow = p.out + static_cast<size_t>(row) * kHeads * kDv;
    for (int e = threadIdx.x; e < kHeads * vecs; e += kThreads) {
      const int h = e / vecs, dv = e - h * vecs;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = 0; r < S; ++r) {
        const float4 x = *reinterpret_cast<const float4*>(recv + (r * kHeads + h) * kStride + 4 * dv);
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
      *reinterpret_cast<float4*>(orow + h * kDv + 4 * (v0 + dv)) = acc;
      if (p.out_bf16 != nullptr) {
        const uint32_t lo = pack_bf16(acc.x, acc.y), hi = pack_bf16(acc.z, acc.w);
        *reinterpret_cast<uint2*>(p.out_bf16 + static_cast<size_t>(row) * kHeads * kDv + h * kDv + 4 * (v0 + dv)) =
            make_uint2(lo, hi);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Splits of the K slots per query (at most kMaxSplits, the CTAs of one
// cluster) so that rows * splits fills ~148 SMs once.
int attend_splits(int rows, int top_k) {
  const int chunks = (top_k + kChunk - 1) / kChunk;
  int best = 1;
  for (int s = 1; s <= chunks && s <= kMaxSplits; ++s) {
    if (chunks % s == 0 && static_cast<long long>(rows) * s <= 148) best = s;
  }
  return best;
}

cudaError_t launch_attend(const AttendArgs& a, cudaStream_t stream) {
  const int rows = a.batch * a.n_q;
  if (rows == 0) return cudaSuccess;
  const int splits = attend_splits(rows, a.top_k);
  CUtensorMap qmap, kvmap;
  cudaError_t e = make_tmap_bf16_2d(&qmap, a.q, kDq, static_cast<uint64_t>(rows) * kHeads, kDq * 2, 64, kHeads);
  if (e != cudaSuccess) return e;
  // every cache row of every sequence, one 64-dim box per row (gather4 takes four rows at a time)
  e = make_tmap_bf16_2d(&kvmap, a.kv, kDq, static_cast<uint64_t>(a.batch) * a.kv_stride, kDq * 2, 64, 1);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(sga_attend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes));
  if (e != cudaSuccess) return e;
  AttendParams p;
  p.kv = a.kv;
  p.idx = a.idx;
  p.gate = a.gate;
  p.out = a.out;
  p.out_bf16 = a.out_bf16;
  p.status = a.status;
  p.n_q = a.n_q;
  p.kv_stride = a.kv_stride;
  p.top_k = a.top_k;
  p.splits = splits;
  p.chunks_per_split = (a.top_k + kChunk - 1) / kChunk / splits;
  p.scale_log2 = static_cast<float>(0.07216878364870322 * 1.4426950408889634);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(rows * splits));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, sga_attend_kernel, qmap, kvmap, p);
}

}  // namespace sga
