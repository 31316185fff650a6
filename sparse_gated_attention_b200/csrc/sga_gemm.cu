// Weight-streaming GEMM for the layer's projections (the contractions either
// side of the hot path; archdb "A.X K2" attention and gate fields):
//
//   Y[b][n][m] = sum_k X[n][b, k] W[b][m][k]     W row-major [m][k] (K-major), or
//   Y[b][n][m] = sum_k X[n][b, k] W[b][k][m]     W row-major [k][m] (MN-major)
//
// for `batch` independent weight matrices (one per head for W_UK and W_UV, one
// for the packed projections).  With 32 new tokens the weights are the whole
// cost (230 MB for one layer against 2.3 MB of activations), so the design is
// a weight stream:
//   * the weights are the M = 128 operand, read once through a TMA ring whose
//     stages hold 128 x 128 tiles as two 128 x 64 boxes (128-byte swizzle;
//     MN-major weights as 64-wide strips), so one barrier round trip moves
//     32 KB of weights; the tokens are N (padded to 16, at most 128 per work
//     item);
//   * a work item is (batch, 128-row tile, token block, K split); a persistent
//     grid walks the items, and split K keeps every SM streaming when there are
//     fewer tiles than SMs (its partial sums go to the workspace and the
//     consumer adds them in split order);
//   * warp 0 issues the TMA loads (the weight part of the first stages before
//     the programmatic-launch wait: weights do not depend on the previous
//     kernel), warp 1 issues tcgen05.mma (kind::f16, bf16 in, fp32 in TMEM),
//     warps 2-5 move each finished accumulator out of TMEM: fp32 partials, or
//     bf16 straight into the consumer's layout.  Two 128-column accumulators
//     let one item's epilogue overlap the next item's mainloop.
#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace sga {
namespace {

constexpr int kGM = 128;                    // weight rows per tile: MMA M
constexpr int kGBox = 64;                   // K elements per 128-byte box row
constexpr int kGStrip = 2 * kGBox;          // K elements per ring stage
constexpr int kGHalf = kGM * 128;           // one 128 x 64 weight box: 16 KB
constexpr int kGABytes = 2 * kGHalf;        // the weights of one stage: 32 KB
constexpr int kGRingBytes = 208 * 1024;     // 5 stages at 32 tokens, 3 at 128
constexpr int kGMaxStages = 16;
constexpr int kGThreads = 192;
constexpr int kGAccCols = kGemmMaxN;        // one accumulator: 128 lanes x up to 128 columns
constexpr int kGNumBars = 2 * kGMaxStages + 4 + 1;
constexpr size_t kGSmem = 1024 + kGRingBytes + kGNumBars * 8 + 16;
static_assert(kGSmem <= 232448, "shared memory budget");

struct GemmParams {
  int m, n, k, batch, splits, m_tiles, n_blocks, k_strips, n_pad;
  int stages, stage_bytes;  // the ring: as many stages of (weight strip + token strip) as fit
  long long items;
  int w_rows_per_batch;  // K-major: rows of W per batch (m); MN-major: rows per batch (k)
  int x_col_per_batch;   // element offset of batch b's K range within an X row
  float* part;           // fp32 output: part[split][col][m_total] (split stride part_split)
  long long part_split;
  int part_ld;
  uint16_t* out;         // bf16 output: out[col * out_ld + b * out_boff + m]
  int out_ld, out_boff;
};

struct Item {
  int b, t, nb, s, ks0, ks1;
};

__device__ __forceinline__ Item decode_item(const GemmParams& p, long long j, int* status) {
  Item it;
  it.s = static_cast<int>(j % p.splits);
  long long r = j / p.splits;
  it.nb = static_cast<int>(r % p.n_blocks);
  r /= p.n_blocks;
  it.t = static_cast<int>(r % p.m_tiles);
  it.b = static_cast<int>(r / p.m_tiles);
  it.ks0 = static_cast<int>(static_cast<long long>(p.k_strips) * it.s / p.splits);
  it.ks1 = static_cast<int>(static_cast<long long>(p.k_strips) * (it.s + 1) / p.splits);
  SGA_DCHECK(status, it.ks0 < it.ks1 && it.t * kGM < p.m && it.nb * kGemmMaxN < p.n && it.b < p.batch);
  return it;
}

template <bool kMnMajor>
__global__ void __launch_bounds__(kGThreads, 1)
    sga_gemm_kernel(const __grid_constant__ CUtensorMap wmap, const __grid_constant__ CUtensorMap xmap, GemmParams p,
                    int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t ring = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGRingBytes);
  const uint32_t bar0 = smem_u32(bars);
  const int stages = p.stages;
  const uint32_t stage_bytes = static_cast<uint32_t>(p.stage_bytes);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kGMaxStages + s); };
  auto accfull = [&](int a) { return bar0 + 8u * (2 * kGMaxStages + a); };
  auto accempty = [&](int a) { return bar0 + 8u * (2 * kGMaxStages + 2 + a); };
  const uint32_t done_bar = bar0 + 8u * (2 * kGMaxStages + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kGNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accfull(a), 1);
      mbar_init(accempty(a), 4);  // one arrival per epilogue warp
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&wmap);
    prefetch_tmap(&xmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kGAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t b_half = static_cast<uint32_t>(p.n_pad) * 128u;  // one 64-wide token box
  const uint32_t b_bytes = 2u * b_half;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights stream through once
      const uint64_t pol_x = policy_evict_last();   // tokens are re-read by every tile
      auto load_w = [&](int st, const Item& it, int ks) {
        const uint32_t a_dst = ring + st * stage_bytes;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if constexpr (kMnMajor) {
            // per 64 k rows, two 64-wide strips of the m tile (8 KB each)
            const int y = it.b * p.w_rows_per_batch + ks * kGStrip + h * kGBox;
            tma_load_2d(a_dst + h * kGHalf, &wmap, full(st), it.t * kGM, y, pol_w);
            tma_load_2d(a_dst + h * kGHalf + kGHalf / 2, &wmap, full(st), it.t * kGM + 64, y, pol_w);
          } else {
            tma_load_2d(a_dst + h * kGHalf, &wmap, full(st), ks * kGStrip + h * kGBox,
                        it.b * p.w_rows_per_batch + it.t * kGM, pol_w);
          }
        }
      };
      auto load_x = [&](int st, const Item& it, int ks) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tma_load_2d(ring + st * stage_bytes + kGABytes + h * b_half, &xmap, full(st),
                      it.b * p.x_col_per_batch + ks * kGStrip + h * kGBox, it.nb * kGemmMaxN, pol_x);
      };
      // This CTA's (item, K strip) sequence.
      long long j = blockIdx.x;
      Item it{};
      int ks = 0;
      bool valid = j < p.items;
      if (valid) {
        it = decode_item(p, j, status);
        ks = it.ks0;
      }
      auto advance = [&]() {
        if (++ks == it.ks1) {
          j += gridDim.x;
          valid = j < p.items;
          if (valid) {
            it = decode_item(p, j, status);
            ks = it.ks0;
          }
        }
      };
      // The weights do not depend on the previous kernel: the first stages'
      // weight strips are issued before waiting for it, their token strips after.
      Item pre_it[kGMaxStages];
      int pre_ks[kGMaxStages];
      int n_pre = 0;
      while (valid && n_pre < stages) {
        mbar_arrive_expect_tx(full(n_pre), kGABytes + b_bytes);
        load_w(n_pre, it, ks);
        pre_it[n_pre] = it;
        pre_ks[n_pre] = ks;
        ++n_pre;
        advance();
      }
      grid_dependency_wait();
      grid_launch_dependents();
      for (int i = 0; i < n_pre; ++i) load_x(i, pre_it[i], pre_ks[i]);
      long long n_issued = n_pre;
      int st = n_pre % stages;
      uint32_t ph = n_pre == stages ? 1u : 0u;
      bool ok = true;
      while (valid) {
        if (!mbar_wait(empty(st), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full(st), kGABytes + b_bytes);
        load_w(st, it, ks);
        load_x(st, it, ks);
        ++n_issued;
        if (++st == stages) {
          st = 0;
          ph ^= 1u;
        }
        advance();
      }
      if (!ok) {
        record_status(status, kStatusTimeout);
        *abort_flag = 1;
        volatile int never = 0;
        for (long long m = (n_issued > stages ? n_issued - stages : 0); m < n_issued; ++m)
          mbar_wait(full(static_cast<int>(m % stages)), static_cast<uint32_t>((m / stages) & 1), &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kGM, p.n_pad, kMnMajor, false);
      int st = 0;
      uint32_t ph = 0;
      long long n_items = 0;
      bool ok = true;
      for (long long j = blockIdx.x; j < p.items && ok; j += gridDim.x) {
        const Item it = decode_item(p, j, status);
        const int acc = static_cast<int>(n_items & 1);
        if (!mbar_wait(accempty(acc), static_cast<uint32_t>((n_items >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t d = tmem_base + static_cast<uint32_t>(acc * kGAccCols);
        for (int ks = it.ks0; ks < it.ks1; ++ks) {
          if (!mbar_wait(full(st), ph, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = ring + st * stage_bytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // 16 K elements per MMA: 32 bytes along a K-major row, or 16 rows of an MN-major strip;
            // MMAs 0-3 read the stage's first 64-wide box, 4-7 its second
            const uint32_t ah = a + static_cast<uint32_t>((kk >> 2) * kGHalf);
            const uint64_t adesc = kMnMajor ? sdesc_sw128(ah + (kk & 3) * 2048, kGHalf / 2, 1024)
                                            : sdesc_sw128(ah + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = sdesc_sw128(a + kGABytes + (kk >> 2) * b_half + (kk & 3) * 32, 16, 1024);
            mma_bf16(d, adesc, bdesc, idesc, (ks > it.ks0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(empty(st));
          if (++st == stages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(accfull(acc));
        ++n_items;
      }
      if (!ok) {
        record_status(status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lane quarter w % 4: weight row m = 32 (w % 4) + lane of
    // the tile, 32 token columns per load.
    const int quarter = warp & 3;
    long long n_items = 0;
    for (long long j = blockIdx.x; j < p.items; j += gridDim.x) {
      const Item it = decode_item(p, j, status);
      const int acc = static_cast<int>(n_items & 1);
      if (!mbar_wait(accfull(acc), static_cast<uint32_t>((n_items >> 1) & 1), abort_flag)) {
        record_status(status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const int m = it.t * kGM + quarter * 32 + lane;
      for (int c = 0; c < p.n_pad; c += 32) {
        float v[32];
        tmem_ld32(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(acc * kGAccCols + c),
                  v);
        if (m < p.m) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int col = it.nb * kGemmMaxN + c + i;
            if (col < p.n) {
              if (p.out) {
                p.out[static_cast<size_t>(col) * p.out_ld + static_cast<size_t>(it.b) * p.out_boff + m] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(v[i]));
              } else {
                p.part[static_cast<size_t>(it.s) * p.part_split + static_cast<size_t>(col) * p.part_ld +
                       static_cast<size_t>(it.b) * p.m + m] = v[i];
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty(acc));
      ++n_items;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kGAccCols);
  }
}

}  // namespace

// The K split with the least time on the busiest SM, counted in ring stages
// (32 KB of weights each): ceil(items / SMs) items of ceil(k_strips / S) stages, plus the
// fp32 partial sums each extra split writes and its consumer reads back, spread
// over the SMs.  S is at most 8; ties go to the smaller S.
int gemm_splits(int m, int n, int k, int batch, int num_sms) {
  const long long tiles = static_cast<long long>(batch) * ((m + kGM - 1) / kGM) * ((n + kGemmMaxN - 1) / kGemmMaxN);
  const int k_strips = (k + kGStrip - 1) / kGStrip;
  const double partial_strips = 8.0 * n * m * batch / (static_cast<double>(kGABytes) * num_sms);
  int best = 1;
  double best_cost = -1.0;
  for (int s = 1; s <= 8 && s <= k_strips; ++s) {
    const long long waves = (tiles * s + num_sms - 1) / num_sms;
    const double cost = static_cast<double>(waves * ((k_strips + s - 1) / s)) + (s - 1) * partial_strips;
    if (best_cost < 0.0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

cudaError_t launch_gemm(const GemmArgs& a, int num_sms, cudaStream_t stream) {
  if (a.m < 1 || a.n < 1 || a.k < 1 || a.batch < 1 || a.splits < 1) return cudaErrorInvalidValue;
  if ((a.out == nullptr) == (a.part == nullptr)) return cudaErrorInvalidValue;
  if (a.out && a.splits != 1) return cudaErrorInvalidValue;
  GemmParams p;
  p.m = a.m;
  p.n = a.n;
  p.k = a.k;
  p.batch = a.batch;
  p.splits = a.splits;
  p.m_tiles = (a.m + kGM - 1) / kGM;
  p.n_blocks = (a.n + kGemmMaxN - 1) / kGemmMaxN;
  p.k_strips = (a.k + kGStrip - 1) / kGStrip;
  if (a.splits > p.k_strips) return cudaErrorInvalidValue;
  // A stage spans 128 of K.  Past the end of K a K-major weight box reads zeros,
  // but an MN-major one, or the token box of a batch other than the last, would
  // read the next batch's rows: those shapes need K a multiple of 128.
  if ((a.w_mn_major || a.batch > 1) && a.k % kGStrip != 0) return cudaErrorInvalidValue;
  const int n_in_block = a.n < kGemmMaxN ? a.n : kGemmMaxN;
  p.n_pad = (n_in_block + 15) / 16 * 16;
  p.stage_bytes = kGABytes + 2 * p.n_pad * 128;  // a multiple of 4 KB: every box keeps the 1 KB swizzle alignment
  p.stages = kGRingBytes / p.stage_bytes;
  if (p.stages > kGMaxStages) p.stages = kGMaxStages;
  p.items = static_cast<long long>(a.batch) * p.m_tiles * p.n_blocks * a.splits;
  p.w_rows_per_batch = a.w_mn_major ? a.k : a.m;
  p.x_col_per_batch = a.x_col_per_batch;
  p.part = a.part;
  p.part_split = static_cast<long long>(a.n) * a.batch * a.m;
  p.part_ld = a.batch * a.m;
  p.out = a.out;
  p.out_ld = a.out_ld;
  p.out_boff = a.out_boff;
  CUtensorMap wmap, xmap;
  cudaError_t e;
  if (a.w_mn_major) {
    // rows: batch * k (k index), columns: m; box 64 m x 64 k rows
    e = make_tmap_bf16_2d(&wmap, a.w, a.m, static_cast<uint64_t>(a.batch) * a.k, static_cast<uint64_t>(a.m) * 2, 64,
                          kGBox);
  } else {
    // rows: batch * m, columns: k; box 64 k x 128 m rows
    e = make_tmap_bf16_2d(&wmap, a.w, a.k, static_cast<uint64_t>(a.batch) * a.m, static_cast<uint64_t>(a.k) * 2, 64,
                          kGM);
  }
  if (e != cudaSuccess) return e;
  // tokens: rows n, columns x_ld elements; box 64 x n_pad rows
  e = make_tmap_bf16_2d(&xmap, a.x, a.x_ld, a.n, static_cast<uint64_t>(a.x_ld) * 2, 64, static_cast<uint32_t>(p.n_pad));
  if (e != cudaSuccess) return e;
  auto kernel = a.w_mn_major ? sga_gemm_kernel<true> : sga_gemm_kernel<false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kGSmem));
  if (e != cudaSuccess) return e;
  const long long grid = p.items < num_sms ? p.items : num_sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kGThreads);
  cfg.dynamicSmemBytes = kGSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, wmap, xmap, p, a.status);
}

}  // namespace sga
