// Step 1: the DSA-style indexer (archdb "A.X K2", token-selection field: 64
// indexer heads of dim 128, ReLU-scored; indexer-key-width field: 128 per token).
//
//   scores[row, s] = sum_j w[row, j] * max(0, q_idx[row, j, :] . k_idx[b, s, :]),  s <= t
//
// Design (decode is HBM-bound: the index key of every past token is read once
// and is ~93% of the bytes of the whole path at 128K context):
//   * A persistent grid, one CTA per SM, walks a contiguous range of
//     (query, 128-key tile) work items.
//   * Warp 0 streams 32 KB tiles of k_idx with TMA (128-byte swizzle, L2
//     evict-first) through a 5-stage shared-memory ring, and the query's
//     64 x 128 indexer matrix into a double buffer when the query changes.
//     bf16 keys: a tile is 128 keys x 128 dims.  E4M3 keys (the FP8 cache of
//     archdb "A.X K2", pretraining-precision field; nlp.com.ai "A.X K2 FP8"):
//     a tile is 256 keys (two M = 128 halves), so one barrier round trip per
//     stage covers as many bytes as in bf16.
//   * Warp 1 issues tcgen05.mma (M = 128 keys, N = 64 heads, K = 128 dims in 8
//     kind::f16 steps of 16, or 4 kind::f8f6f4 steps of 32 per half) into one
//     of eight 64-column (bf16) or four 128-column (E4M3) TMEM accumulators.
//   * Warps 2-9, two groups of four that take alternate tiles (one warp per
//     TMEM lane quarter in each; a thread takes one key per 128-key half),
//     read a key's 64 head dots with tcgen05.ld,
//     apply ReLU, the per-head weight and the head sum in fp32, mask s > t and
//     store the score (32 consecutive keys per warp: one 128-byte store).
//     When the caller asks for it, they also count each score's top 12 order
//     bits into a per-query shared-memory histogram (one per group) that is
//     added to global memory when the query changes: the first level of the
//     top-k radix select, computed while the scores are still in registers.
#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace sga {
namespace {

constexpr int kKeys = 128;    // keys per tile: MMA M
constexpr int kDim = 128;     // indexer dim: MMA K
constexpr int kHeads = 64;    // indexer heads: MMA N
constexpr int kABox = kKeys * 128;  // one 128-byte-wide column strip of a tile (16 KB)
constexpr int kQBox = kHeads * 128;  // one 128-byte-wide column strip of a query's matrix (8 KB)
constexpr int kTmemCols = 512;  // TMEM accumulators fill all 512 columns
constexpr int kEpiGroups = 2;   // epilogue warp groups, taking alternate tiles
constexpr int kThreads = 64 + kEpiGroups * 128;
constexpr int kThrWarp = 2 + 4 * kEpiGroups;  // the candidate threshold warp (candidate mode only)
constexpr int kCandThreads = kThreads + 32;
constexpr int kHistBytes = kTopkHistBins * 4;
constexpr int kEpiThreads = 128;

// bf16 keys: a key row is 256 B, two 128-byte strips; K = 128 in 8 MMA steps of
// 16; a tile is 128 keys.  E4M3 keys: a key row is one 128-byte strip; K = 128
// in 4 MMA steps of 32; a tile is 256 keys (two M = 128 halves), so both tiles
// are 32 KB and one barrier round trip per stage covers the same bytes.
template <bool kFp8>
struct IndexCfg {
  static constexpr int kStrips = kFp8 ? 1 : 2;        // 128-byte strips per key (and query) row
  static constexpr int kStripElems = kFp8 ? 128 : 64;  // elements per strip
  static constexpr int kHalves = kFp8 ? 2 : 1;         // 128-key halves per tile (one MMA M each)
  static constexpr int kTileKeys = kKeys * kHalves;
  static constexpr int kStages = 5;
  static constexpr int kAStage = kStrips * kABox * kHalves;  // 32 KB
  static constexpr int kQBuf = kStrips * kQBox;
  static constexpr int kKSteps = kFp8 ? 4 : 8;         // 32-byte K steps per tile
  static constexpr int kAccCols = kHeads * kHalves;    // one tile's accumulator
  static constexpr int kAcc = kTmemCols / kAccCols;    // 8 (bf16) or 4 (E4M3) tiles in flight
  static_assert((kAcc & (kAcc - 1)) == 0, "the epilogue indexes accumulators with a mask");
  static constexpr int kNumBars = 2 * kStages + 4 + 2 * kAcc + 1;
  static constexpr size_t kSmemBytes =
      1024 + kStages * kAStage + 2 * kQBuf + kEpiGroups * kHistBytes + kNumBars * 8 + 32;
  static constexpr uint32_t kIdesc = kFp8 ? idesc_e4m3_f32(kKeys, kHeads) : idesc_bf16_f32(kKeys, kHeads, false, false);
};
static_assert(IndexCfg<false>::kSmemBytes <= 232448 && IndexCfg<true>::kSmemBytes <= 232448, "shared memory budget");

struct IndexParams {
  const uint16_t* w;
  const int32_t* q_pos;
  float* scores;
  uint32_t* hist;    // [rows][kTopkHistBins] or null
  uint64_t* cand;    // candidate mode: [rows][kv_stride] selection candidates
  uint32_t* cand_n;  // candidate mode: [rows][kCandNStride]
  int* status;
  int n_q, kv_stride, tiles_per_row, top_k;
  long long total_tiles;
};

// A bin below which no key of a row can be among its top_k, from the row's
// global histogram as far as it has been counted: the highest bin b with at
// least top_k counted keys in bins >= b, or 0 while fewer are counted.  Every
// counted key is a real key of the row, so at least top_k keys of the row are
// larger than any key in a lower bin.  One warp reads the bins from the top,
// 1,024 per round (lane l: 32 bins, lane 0 the highest), and stops at the
// round that reaches top_k.
__device__ __noinline__ uint32_t candidate_threshold(const uint32_t* hrow, uint32_t top_k) {
  const int lane = threadIdx.x & 31;
  uint32_t carry = 0;
  for (int round = 0; round < kTopkHistBins / 1024; ++round) {
    const int base = kTopkHistBins - 1024 * (round + 1) + 32 * (31 - lane);  // this lane's lowest bin
    const uint4* hp = reinterpret_cast<const uint4*>(hrow + base);
    uint32_t h[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 v = __ldcg(hp + i);
      h[4 * i] = v.x;
      h[4 * i + 1] = v.y;
      h[4 * i + 2] = v.z;
      h[4 * i + 3] = v.w;
    }
    uint32_t sum = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) sum += h[k];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t hi = carry + incl, lo = hi - sum;  // counted keys above and at this lane's bins
    uint32_t b = 0;
    if (lo < top_k && top_k <= hi) {
      uint32_t run = lo;
      bool found = false;
#pragma unroll
      for (int k = 31; k >= 0; --k) {
        run += h[k];
        if (!found && run >= top_k) {
          b = static_cast<uint32_t>(base + k);
          found = true;
        }
      }
    }
    const uint32_t hit = __ballot_sync(0xFFFFFFFFu, lo < top_k && top_k <= hi);
    if (hit != 0u) return __shfl_sync(0xFFFFFFFFu, b, __ffs(hit) - 1);
    carry += __shfl_sync(0xFFFFFFFFu, incl, 31);
  }
  return 0u;
}


// Walks work items j = (query row, 128-key tile) in order: one division at
// the start, then a key step per item; the query position is read only when
// the row changes.
template <int kTileKeys>
struct TileCursor {
  int row, key0, t;
  __device__ __forceinline__ void start(const IndexParams& p, long long j) {
    row = static_cast<int>(j / p.tiles_per_row);
    key0 = static_cast<int>(j % p.tiles_per_row) * kTileKeys;
    t = __ldg(p.q_pos + row);
  }
  // Moves to item j + 1; `more` is false after the last item of the range.
  __device__ __forceinline__ void next(const IndexParams& p, bool more) {
    key0 += kTileKeys;
    if (key0 >= p.tiles_per_row * kTileKeys) {
      key0 = 0;
      ++row;
      if (more) t = __ldg(p.q_pos + row);
    }
  }
  __device__ __forceinline__ bool bad_position(const IndexParams& p) const { return t < 0 || t >= p.kv_stride; }
  // False for tiles past the query position or rows whose position is invalid.
  __device__ __forceinline__ bool live(const IndexParams& p) const { return !bad_position(p) && key0 <= t; }
};

// kCand: instead of scores, every key that can still be among its row's top_k
// is appended to the row's candidate list (order key, position), and a
// threshold warp keeps a bin below which keys are dropped, from the row's
// global histogram as counted so far (the epilogue adds its counts every 8
// tiles).  The candidate mode needs the histogram.
template <bool kFp8, bool kCand>
__global__ void __launch_bounds__(kCand ? kCandThreads : kThreads, 1)
    sga_index_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                     IndexParams p) {
  using C = IndexCfg<kFp8>;
  constexpr int kStages = C::kStages, kAStage = C::kAStage, kQBuf = C::kQBuf, kNumBars = C::kNumBars;
  constexpr int kAcc = C::kAcc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t a_base = smem_u32(smem);
  const uint32_t q_base = a_base + kStages * kAStage;
  uint32_t* hist_s = reinterpret_cast<uint32_t*>(smem + kStages * kAStage + 2 * kQBuf);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kAStage + 2 * kQBuf + kEpiGroups * kHistBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto qfull = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  auto qempty = [&](int s) { return bar0 + 8u * (2 * kStages + 2 + s); };
  auto accfull = [&](int s) { return bar0 + 8u * (2 * kStages + 4 + s); };
  auto accempty = [&](int s) { return bar0 + 8u * (2 * kStages + 4 + kAcc + s); };
  const uint32_t done_bar = bar0 + 8u * (2 * kStages + 4 + 2 * kAcc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // candidate mode: the row the epilogue works on, the groups that have
  // finished, and the threshold warp's latest (row << 32 | bin)
  int* row_s = reinterpret_cast<int*>(tmem_slot + 2);
  int* done_s = row_s + 1;
  volatile unsigned long long* thr_tag = reinterpret_cast<volatile unsigned long long*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(qfull(s), 1);
      mbar_init(qempty(s), 1);
    }
    for (int s = 0; s < kAcc; ++s) {
      mbar_init(accfull(s), 1);
      mbar_init(accempty(s), 4 * 32);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    *row_s = -1;
    *done_s = 0;
    *thr_tag = ~0ull;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Set-up above overlaps the previous kernel on the stream; inputs are read below.
  grid_dependency_wait();
  grid_launch_dependents();

  const long long j0 = p.total_tiles * blockIdx.x / gridDim.x;
  const long long j1 = p.total_tiles * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      long long n = 0, qc = 0;
      int st = 0;         // ring stage of tile n
      uint32_t ph = 0;    // phase parity of that stage's current use
      int cur_row = -1;
      bool ok = true;
      TileCursor<C::kTileKeys> cur;
      if (j0 < j1) cur.start(p, j0);
      for (long long j = j0; j < j1; cur.next(p, ++j < j1)) {
        if (!cur.live(p)) {
          if (cur.bad_position(p)) record_status(p.status, kStatusDeviceArg);
          continue;
        }
        const int row = cur.row, key0 = cur.key0;
        if (row != cur_row) {
          const int slot = static_cast<int>(qc & 1);
          if (!mbar_wait(qempty(slot), static_cast<uint32_t>((qc >> 1) & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(qfull(slot), kQBuf);
#pragma unroll
          for (int b = 0; b < C::kStrips; ++b)
            tma_load_2d(q_base + slot * kQBuf + b * kQBox, &qmap, qfull(slot), b * C::kStripElems, row * kHeads,
                        pol_keep);
          ++qc;
          cur_row = row;
        }
        if (!mbar_wait(empty(st), ph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(full(st), kAStage);
        const int y = (row / p.n_q) * p.kv_stride + key0;
#pragma unroll
        for (int b = 0; b < C::kStrips; ++b)
          tma_load_2d(a_base + st * kAStage + b * kABox, &kmap, full(st), b * C::kStripElems, y, pol_stream);
        // (an E4M3 tile is one box of 256 key rows: both halves, 16 KB apart)
        ++n;
        if (++st == kStages) {
          st = 0;
          ph ^= 1u;
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        // Let the copies already issued land before the CTA retires.
        volatile int never = 0;
        for (long long m = (n > kStages ? n - kStages : 0); m < n; ++m)
          mbar_wait(full(static_cast<int>(m % kStages)), static_cast<uint32_t>((m / kStages) & 1), &never);
        for (long long m = (qc > 2 ? qc - 2 : 0); m < qc; ++m)
          mbar_wait(qfull(static_cast<int>(m & 1)), static_cast<uint32_t>((m >> 1) & 1), &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = C::kIdesc;
      // Descriptors are built once and stepped: the start-address field is
      // address / 16, so adding (offset / 16) moves a descriptor by offset bytes.
      const uint64_t a_desc0 = sdesc_sw128(a_base, 16, 1024);
      const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
      long long qc = 0;
      int st = 0, acc = 0;            // ring stage and TMEM accumulator of the next tile
      uint32_t ph = 0, aph = 0;       // their phase parities
      int cur_row = -1, cur_q = 0;
      bool ok = true;
      TileCursor<C::kTileKeys> cur;
      if (j0 < j1) cur.start(p, j0);
      for (long long j = j0; j < j1 && ok; cur.next(p, ++j < j1)) {
        if (!cur.live(p)) continue;
        const int row = cur.row;
        if (row != cur_row) {
          if (cur_row >= 0) mma_commit(qempty(cur_q));  // frees the previous query's buffer
          const int slot = static_cast<int>(qc & 1);
          if (!mbar_wait(qfull(slot), static_cast<uint32_t>((qc >> 1) & 1), abort_flag)) {
            ok = false;
            break;
          }
          cur_q = slot;
          ++qc;
          cur_row = row;
        }
        if (!mbar_wait(accempty(acc), aph ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        if (!mbar_wait(full(st), ph, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t b_desc = q_desc0 + static_cast<uint64_t>((cur_q * kQBuf) >> 4);
#pragma unroll
        for (int hh = 0; hh < C::kHalves; ++hh) {
          const uint32_t d = tmem_base + static_cast<uint32_t>(acc * C::kAccCols + hh * kHeads);
          const uint64_t a_desc = a_desc0 + static_cast<uint64_t>((st * kAStage + hh * kABox) >> 4);
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            // 32-byte K steps: four per 128-byte strip
            const uint64_t a_off = static_cast<uint64_t>(((k >> 2) * kABox + (k & 3) * 32) >> 4);
            const uint64_t b_off = static_cast<uint64_t>(((k >> 2) * kQBox + (k & 3) * 32) >> 4);
            if constexpr (kFp8)
              mma_e4m3(d, a_desc + a_off, b_desc + b_off, idesc, k > 0 ? 1u : 0u);
            else
              mma_bf16(d, a_desc + a_off, b_desc + b_off, idesc, k > 0 ? 1u : 0u);
          }
        }
        mma_commit(empty(st));
        mma_commit(accfull(acc));
        if (++st == kStages) {
          st = 0;
          ph ^= 1u;
        }
        if (++acc == kAcc) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      // Every MMA this thread issued has finished once done_bar flips.
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never);
    }
  } else if (kCand && warp == kThrWarp) {
    // ------------------------------------------------------------ candidate threshold
    // Every few microseconds: the row the epilogue works on, that row's global
    // histogram as counted so far, and, when it rises, the threshold published
    // for the epilogue (which drops keys in lower bins).  Ends when both
    // epilogue groups have finished, or after the wait budget.
    if constexpr (kCand) {
      const long long t_start = clock64();
      int trow = -1;
      uint32_t tbin = 0;
      while (*reinterpret_cast<volatile int*>(done_s) < kEpiGroups && clock64() - t_start < kWaitBudgetCycles) {
        const int r = *reinterpret_cast<volatile int*>(row_s);
        if (r >= 0) {
          if (r != trow) {
            trow = r;
            tbin = 0;
          }
          const uint32_t b =
              candidate_threshold(p.hist + static_cast<size_t>(r) * kTopkHistBins, static_cast<uint32_t>(p.top_k));
          if (b > tbin) {
            tbin = b;
            if (lane == 0) *thr_tag = (static_cast<unsigned long long>(static_cast<uint32_t>(r)) << 32) | b;
          }
        }
        // about 3 us until the next look, in short sleeps so the CTA is not held up at its end
        for (int i = 0; i < 8 && *reinterpret_cast<volatile int*>(done_s) < kEpiGroups; ++i) __nanosleep(400);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Two groups of four warps take alternate tiles (group g reads the
    // accumulators of its parity), each with its own histogram, so a group has
    // two tile periods per tile.
    const int group = (warp - 2) >> 2;
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31 (warp % 4 rule)
    const int et = threadIdx.x - 64 - kEpiThreads * group;
    const int bar_id = 1 + group;
    uint32_t* hist_g = hist_s + group * kTopkHistBins;
    const bool with_hist = kCand || p.hist != nullptr;
    int an = 0;  // live tiles seen (both groups' ones): accumulator an % kAcc
    int cur_row = -1;
    float wv[kHeads];  // the row's head weights
    // Candidate mode: every 8 of its tiles the group adds its counts to the
    // row's global histogram (each bin read and cleared atomically, so no
    // barrier), and before each tile it takes the threshold warp's latest bin
    // for the row; keys in lower bins are dropped.  A warp's candidates of one
    // tile half are stored one group tile later: the counter update's result
    // is read only then, so its round trip to L2 overlaps the next tile.
    uint32_t thr = 0;  // bins below thr hold no key of the row's top_k
    int gtiles = 0;
    uint32_t pend_m[C::kHalves], pend_base[C::kHalves];
    uint64_t pend_val[C::kHalves];
    int pend_row = 0;
#pragma unroll
    for (int hh = 0; hh < C::kHalves; ++hh) pend_m[hh] = 0u;
    auto store_pending = [&]() {
#pragma unroll
      for (int hh = 0; hh < C::kHalves; ++hh) {
        if (pend_m[hh] != 0u) {
          const uint32_t base = __shfl_sync(0xFFFFFFFFu, pend_base[hh], 0);
          const uint32_t below = pend_m[hh] & ((1u << lane) - 1u);
          const uint32_t slot = base + static_cast<uint32_t>(__popc(below));
          const bool mine = (pend_m[hh] >> lane) & 1u;
          SGA_DCHECK(p.status, !mine || slot < static_cast<uint32_t>(p.kv_stride));
          if (mine && slot < static_cast<uint32_t>(p.kv_stride))
            p.cand[static_cast<size_t>(pend_row) * p.kv_stride + slot] = pend_val[hh];
          pend_m[hh] = 0u;
        }
      }
    };
    // Adds the shared histogram of `r` to global memory and clears it.
    auto flush_hist = [&](int r) {
      named_barrier(bar_id, kEpiThreads);
      for (int b = et; b < kTopkHistBins; b += kEpiThreads) {
        const uint32_t v = hist_g[b];
        if (v) {
          atomicAdd(p.hist + static_cast<size_t>(r) * kTopkHistBins + b, v);
          hist_g[b] = 0;
        }
      }
      named_barrier(bar_id, kEpiThreads);
    };
    if (with_hist) {
      for (int b = et; b < kTopkHistBins; b += kEpiThreads) hist_g[b] = 0;
      named_barrier(bar_id, kEpiThreads);
    }
    TileCursor<C::kTileKeys> cur;
    if (j0 < j1) cur.start(p, j0);
    for (long long j = j0; j < j1; cur.next(p, ++j < j1)) {
      if (!cur.live(p)) continue;
      if ((an & 1) != group) {  // the other group's tile
        ++an;
        continue;
      }
      const int row = cur.row, key0 = cur.key0, t = cur.t;
      if (row != cur_row) {
        if (with_hist && cur_row >= 0) flush_hist(cur_row);
        if constexpr (kCand) {
          thr = 0;
          gtiles = 0;
          if (et == 0) atomicMax(row_s, row);
        }
        const uint4* wp = reinterpret_cast<const uint4*>(p.w + static_cast<size_t>(row) * kHeads);
#pragma unroll
        for (int c = 0; c < kHeads / 8; ++c) {
          const uint4 u = __ldg(wp + c);
          const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            wv[8 * c + 2 * e] = __uint_as_float(x[e] << 16);
            wv[8 * c + 2 * e + 1] = __uint_as_float(x[e] & 0xFFFF0000u);
          }
        }
        cur_row = row;
      }
      const int acc = an & (kAcc - 1);
      if (!mbar_wait(accfull(acc), static_cast<uint32_t>(an / kAcc) & 1u, abort_flag)) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      if constexpr (kCand) {
        store_pending();
        const unsigned long long tv = *thr_tag;
        if (static_cast<uint32_t>(tv >> 32) == static_cast<uint32_t>(row)) thr = max(thr, static_cast<uint32_t>(tv));
      }
      tc_fence_after();
#pragma unroll
      for (int hh = 0; hh < C::kHalves; ++hh) {
        float v[64];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                               static_cast<uint32_t>(acc * C::kAccCols + hh * kHeads);
        tmem_ld64(taddr, v);
        if (hh == C::kHalves - 1) {
          tc_fence_before();
          mbar_arrive(accempty(acc));
        }
        // head sum as four independent chains (one warp per scheduler: the chain
        // latency, not issue, bounds the epilogue); integer-valued inputs keep
        // every partial sum exact, so the order does not change the score
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 64; ++h) ps[h & 3] = fmaf(wv[h], fmaxf(v[h], 0.f), ps[h & 3]);
        const float s = (ps[0] + ps[1]) + (ps[2] + ps[3]);
        const int key = key0 + hh * kKeys + quarter * 32 + lane;
        if constexpr (kCand) {
          // this warp's surviving keys are counted and appended with one
          // counter update.  Keys below the threshold are not counted: every
          // threshold lies at or below the K-th key's bin, and neither a later
          // threshold nor the selection reads the counts of lower bins.
          const uint32_t kb = order_bits(s);
          const bool c = key <= t && (kb >> (32 - kTopkHistBits)) >= thr;
          if (c) atomicAdd(hist_g + (kb >> (32 - kTopkHistBits)), 1u);
          const uint32_t m = __ballot_sync(0xFFFFFFFFu, c);
          pend_m[hh] = m;
          pend_val[hh] = (static_cast<uint64_t>(kb) << 32) | static_cast<uint32_t>(key);
          pend_base[hh] = 0u;
          if (lane == 0 && m != 0u)
            pend_base[hh] =
                atomicAdd(p.cand_n + static_cast<size_t>(row) * kCandNStride, static_cast<uint32_t>(__popc(m)));
          pend_row = row;
        } else if (key <= t) {
          p.scores[static_cast<size_t>(row) * p.kv_stride + key] = s;
          if (with_hist) atomicAdd(hist_g + (order_bits(s) >> (32 - kTopkHistBits)), 1u);
        }
      }
      ++an;
      if (kCand && (++gtiles & 7) == 0) {
        // this thread's bins: eight runs of four, read 16 bytes at a time
        uint32_t* grow = p.hist + static_cast<size_t>(row) * kTopkHistBins;
#pragma unroll
        for (int i = 0; i < kTopkHistBins / (4 * kEpiThreads); ++i) {
          const int b0 = 4 * (et + kEpiThreads * i);
          const uint4 q = *reinterpret_cast<const uint4*>(hist_g + b0);
          if ((q.x | q.y | q.z | q.w) != 0u) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t v = atomicExch(hist_g + b0 + e, 0u);
              if (v != 0u) atomicAdd(grow + b0 + e, v);
            }
          }
        }
      }
    }
    if constexpr (kCand) store_pending();
    if (with_hist && cur_row >= 0) flush_hist(cur_row);
    if (kCand && et == 0) atomicAdd(done_s, 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ============================================================================ prefill
// Many queries per sequence (chunked prefill): a work item is (query block,
// 128-key tile), a block being kQB = 8 consecutive queries of one sequence.
// The tensor core computes D[key, (query, head)] for the block as two N = 256
// halves (4 queries x 64 heads) into two 256-column TMEM accumulators; the
// epilogue drains one half while the tensor core fills the other.  The block's
// queries (the B operand: 128 KB in bf16, 64 KB in E4M3) stay in shared memory
// for all of its tiles, so every key tile serves 8 queries; keys arrive as
// 16 KB strips (128 keys x 128 bytes) through a ring, with an L2 evict-last
// policy because every CTA sweeps the same sequence's keys.  No first-level
// selection histogram is counted here.
constexpr int kQB = 8;                            // queries per block
constexpr int kHalfQ = 4;                         // queries per accumulator
constexpr int kPfN = kHalfQ * kHeads;             // MMA N: 256
constexpr int kPfEpiWarps = 8;                    // two per TMEM lane quarter
constexpr int kPfThreads = 64 + 32 * kPfEpiWarps;  // 320

template <bool kFp8>
struct PrefillCfg {
  static constexpr int kStrips = kFp8 ? 1 : 2;  // 128-byte strips per key / query row
  static constexpr int kStripElems = kFp8 ? 128 : 64;
  static constexpr int kStages = kFp8 ? 8 : 5;  // ring of key strips (16 KB each)
  static constexpr int kQStrip = kPfN * 128;    // one strip of a half's 256 query rows: 32 KB
  static constexpr int kQHalf = kStrips * kQStrip;
  static constexpr int kQBytes = 2 * kQHalf;
  static constexpr int kKSteps = kFp8 ? 4 : 8;
  static constexpr int kWFloats = kHalfQ * kHeads;  // each epilogue warp's four queries' weights
  static constexpr int kWBytes = kPfEpiWarps * kWFloats * 4;
  static constexpr int kNumBars = 2 * kStages + 2 + 4 + 1;
  static constexpr size_t kSmemBytes = 1024 + kStages * kABox + kQBytes + kWBytes + kNumBars * 8 + 16;
  static constexpr uint32_t kIdesc = kFp8 ? idesc_e4m3_f32(kKeys, kPfN) : idesc_bf16_f32(kKeys, kPfN, false, false);
};
static_assert(PrefillCfg<false>::kSmemBytes <= 232448 && PrefillCfg<true>::kSmemBytes <= 232448,
              "shared memory budget");

struct PrefillParams {
  const uint16_t* w;
  const int32_t* q_pos;
  float* scores;
  int* status;
  int n_q, kv_stride, tiles_per_block, blocks_per_seq;
  long long total_items;
};

// Walks work items j = (query block, 128-key tile) in order, re-reading the
// block's positions only when the block changes.  tmax is the largest valid
// position of the block (-1 if none); tiles past it are dead.
struct BlockCursor {
  int blk, key0, seq, row0, nrows, tmax;
  bool bad;  // some row of the block has a position outside [0, L)
  __device__ __forceinline__ void load(const PrefillParams& p) {
    seq = blk / p.blocks_per_seq;
    const int i = blk - seq * p.blocks_per_seq;
    row0 = seq * p.n_q + i * kQB;
    nrows = min(kQB, p.n_q - i * kQB);
    SGA_DCHECK(p.status, nrows > 0 && row0 + nrows <= (seq + 1) * p.n_q);
    tmax = -1;
    bad = false;
    for (int r = 0; r < nrows; ++r) {
      const int t = __ldg(p.q_pos + row0 + r);
      if (t >= 0 && t < p.kv_stride) {
        tmax = max(tmax, t);
      } else {
        bad = true;
      }
    }
  }
  __device__ __forceinline__ void start(const PrefillParams& p, long long j) {
    blk = static_cast<int>(j / p.tiles_per_block);
    key0 = static_cast<int>(j % p.tiles_per_block) * kKeys;
    load(p);
  }
  __device__ __forceinline__ void next(const PrefillParams& p, bool more) {
    key0 += kKeys;
    if (key0 >= p.tiles_per_block * kKeys) {
      key0 = 0;
      ++blk;
      if (more) load(p);
    }
  }
  __device__ __forceinline__ bool live() const { return key0 <= tmax; }
};

// acc += a * b on two fp32 lanes at once (one packed instruction).
__device__ __forceinline__ void ffma2(float2& acc, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 x, y, z;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 y, {%4, %5};\n\t"
      "mov.b64 z, {%0, %1};\n\t"
      "fma.rn.f32x2 z, x, y, z;\n\t"
      "mov.b64 {%0, %1}, z;\n\t}"
      : "+f"(acc.x), "+f"(acc.y)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// sum_j w[j] * max(0, v[j]) over 64 heads, as four independent pairs of
// chains (exact for integer-valued inputs, whatever the order).
__device__ __forceinline__ float weighted_relu_sum(const float (&v)[64], const float* w) {
  const float4* wq = reinterpret_cast<const float4*>(w);
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
  for (int c = 0; c < kHeads / 4; ++c) {
    const float4 wv = wq[c];
    ffma2(acc[(2 * c) & 3], wv.x, wv.y, fmaxf(v[4 * c], 0.f), fmaxf(v[4 * c + 1], 0.f));
    ffma2(acc[(2 * c + 1) & 3], wv.z, wv.w, fmaxf(v[4 * c + 2], 0.f), fmaxf(v[4 * c + 3], 0.f));
  }
  return ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
}

// Score store that should not displace the keys every CTA keeps re-reading from L2.
__device__ __forceinline__ void st_evict_first(float* addr, float v, uint64_t policy) {
  asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(addr), "f"(v), "l"(policy) : "memory");
}

template <bool kFp8>
__global__ void __launch_bounds__(kPfThreads, 1)
    sga_index_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                             PrefillParams p) {
  using C = PrefillCfg<kFp8>;
  constexpr int kStages = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t a_base = smem_u32(smem);
  const uint32_t q_base = a_base + kStages * kABox;
  float* w_s = reinterpret_cast<float*>(smem + kStages * kABox + C::kQBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kABox + C::kQBytes + C::kWBytes);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kStages + s); };
  const uint32_t qfull = bar0 + 8u * (2 * kStages);
  const uint32_t qempty = qfull + 8u;
  auto accfull = [&](int h) { return qfull + 8u * (2 + h); };
  auto accempty = [&](int h) { return qfull + 8u * (4 + h); };
  const uint32_t done_bar = qfull + 8u * 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + C::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(accfull(h), 1);
      mbar_init(accempty(h), kPfEpiWarps);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&kmap);
    prefetch_tmap(&qmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kPfN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependency_wait();
  grid_launch_dependents();

  const long long j0 = p.total_items * blockIdx.x / gridDim.x;
  const long long j1 = p.total_items * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_keys = policy_evict_last();
      const uint64_t pol_q = policy_evict_first();
      long long n = 0;  // strips issued
      int st = 0, qc = 0, seen_blk = -1, q_blk = -1;
      uint32_t ph = 0;
      bool ok = true;
      BlockCursor cur;
      if (j0 < j1) cur.start(p, j0);
      for (long long j = j0; j < j1; cur.next(p, ++j < j1)) {
        if (cur.blk != seen_blk) {
          if (cur.bad) record_status(p.status, kStatusDeviceArg);
          seen_blk = cur.blk;
        }
        if (!cur.live()) continue;
        if (cur.blk != q_blk) {  // the block's queries, once its previous user has finished
          if (!mbar_wait(qempty, static_cast<uint32_t>(qc & 1) ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(qfull, static_cast<uint32_t>(cur.nrows * C::kStrips * kQBox));
          for (int r = 0; r < cur.nrows; ++r)
#pragma unroll
            for (int b = 0; b < C::kStrips; ++b)
              tma_load_2d(q_base + (r / kHalfQ) * C::kQHalf + b * C::kQStrip + (r % kHalfQ) * kQBox, &qmap, qfull,
                          b * C::kStripElems, (cur.row0 + r) * kHeads, pol_q);
          ++qc;
          q_blk = cur.blk;
        }
        const int y = cur.seq * p.kv_stride + cur.key0;
#pragma unroll
        for (int b = 0; b < C::kStrips; ++b) {
          if (!mbar_wait(empty(st), ph ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full(st), kABox);
          tma_load_2d(a_base + st * kABox, &kmap, full(st), b * C::kStripElems, y, pol_keys);
          ++n;
          if (++st == kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        // Let the copies already issued land before the CTA retires.
        volatile int never = 0;
        for (long long m = (n > kStages ? n - kStages : 0); m < n; ++m)
          mbar_wait(full(static_cast<int>(m % kStages)), static_cast<uint32_t>((m / kStages) & 1), &never);
        if (qc > 0) mbar_wait(qfull, static_cast<uint32_t>((qc - 1) & 1), &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = C::kIdesc;
      const uint64_t a_desc0 = sdesc_sw128(a_base, 16, 1024);
      const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
      int st = 0, qc = 0, q_blk = -1;
      uint32_t ph = 0;
      long long tiles = 0;
      bool ok = true;
      BlockCursor cur;
      if (j0 < j1) cur.start(p, j0);
      for (long long j = j0; j < j1 && ok; cur.next(p, ++j < j1)) {
        if (!cur.live()) continue;
        if (cur.blk != q_blk) {
          if (q_blk >= 0) mma_commit(qempty);  // the previous block's queries are free once its MMAs finish
          if (!mbar_wait(qfull, static_cast<uint32_t>(qc & 1), abort_flag)) {
            ok = false;
            break;
          }
          ++qc;
          q_blk = cur.blk;
        }
        int sst[C::kStrips];
#pragma unroll
        for (int b = 0; b < C::kStrips; ++b) {
          if (!mbar_wait(full(st), ph, abort_flag)) ok = false;
          sst[b] = st;
          if (++st == kStages) {
            st = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        const uint32_t tpar = static_cast<uint32_t>(tiles & 1);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(accempty(h), tpar ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem_base + static_cast<uint32_t>(h * kPfN);
#pragma unroll
          for (int k = 0; k < C::kKSteps; ++k) {
            // 32-byte K steps: four per 128-byte strip
            const int b = k >> 2;
            const uint64_t a_desc = a_desc0 + static_cast<uint64_t>((sst[b] * kABox + (k & 3) * 32) >> 4);
            const uint64_t b_desc = q_desc0 + static_cast<uint64_t>((h * C::kQHalf + b * C::kQStrip + (k & 3) * 32) >> 4);
            if constexpr (kFp8)
              mma_e4m3(d, a_desc, b_desc, idesc, k > 0 ? 1u : 0u);
            else
              mma_bf16(d, a_desc, b_desc, idesc, k > 0 ? 1u : 0u);
          }
          mma_commit(accfull(h));
        }
        if (!ok) break;
#pragma unroll
        for (int b = 0; b < C::kStrips; ++b) mma_commit(empty(sst[b]));
        ++tiles;
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
      }
      mma_commit(done_bar);
      volatile int never = 0;
      mbar_wait(done_bar, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // Eight warps, two per TMEM lane quarter: in each half, the first warp of a
    // quarter takes the half's queries 0-1, the second queries 2-3.  Thread =
    // one key (TMEM lane); each warp keeps its four queries' weights in shared
    // memory as fp32.
    const int e = warp - 2;
    const int quarter = warp & 3;
    const int sub = e >> 2;
    float* w_mine = w_s + e * C::kWFloats;  // [h * 2 + qq][64]
    const uint64_t pol_scores = policy_evict_first();
    long long tiles = 0;
    int cur_blk = -1;
    int trow[4] = {-1, -1, -1, -1};
    int rrow[4] = {0, 0, 0, 0};
    BlockCursor cur;
    if (j0 < j1) cur.start(p, j0);
    for (long long j = j0; j < j1; cur.next(p, ++j < j1)) {
      if (!cur.live()) continue;
      if (cur.blk != cur_blk) {
        __syncwarp();
        for (int i = lane; i < C::kWFloats; i += 32) {
          const int s = i >> 6, qi = (s >> 1) * kHalfQ + sub * 2 + (s & 1);
          w_mine[i] = qi < cur.nrows
                          ? bf16_bits_to_float(__ldg(p.w + static_cast<size_t>(cur.row0 + qi) * kHeads + (i & 63)))
                          : 0.f;
        }
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const int qi = (s >> 1) * kHalfQ + sub * 2 + (s & 1);
          int t = -1;
          if (qi < cur.nrows) {
            t = __ldg(p.q_pos + cur.row0 + qi);
            if (t < 0 || t >= p.kv_stride) t = -1;
          }
          trow[s] = t;
          rrow[s] = cur.row0 + qi;
        }
        __syncwarp();
        cur_blk = cur.blk;
      }
      const uint32_t tpar = static_cast<uint32_t>(tiles & 1);
      const int key = cur.key0 + quarter * 32 + lane;
      bool ok = true;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!mbar_wait(accfull(h), tpar, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // one query's 64 head dots at a time (registers: three of the ten
        // warps share a sub-partition, which caps a thread at 168)
        float v[64];
        const uint32_t taddr =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(h * kPfN + sub * 2 * kHeads);
        tmem_ld64(taddr, v);
        const float s0 = weighted_relu_sum(v, w_mine + (h * 2) * kHeads);
        tmem_ld64(taddr + kHeads, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty(h));
        const float s1 = weighted_relu_sum(v, w_mine + (h * 2 + 1) * kHeads);
        if (key <= trow[h * 2])
          st_evict_first(p.scores + static_cast<size_t>(rrow[h * 2]) * p.kv_stride + key, s0, pol_scores);
        if (key <= trow[h * 2 + 1])
          st_evict_first(p.scores + static_cast<size_t>(rrow[h * 2 + 1]) * p.kv_stride + key, s1, pol_scores);
      }
      if (!ok) {
        record_status(p.status, kStatusTimeout);
        *abort_flag = 1;
        break;
      }
      ++tiles;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kPfN);
  }
}

}  // namespace

bool index_uses_prefill(int n_q) { return n_q >= kQB; }

namespace {

cudaError_t launch_prefill(const IndexArgs& a, int num_sms, cudaStream_t stream, const CUtensorMap& kmap,
                           const CUtensorMap& qmap) {
  const int blocks_per_seq = (a.n_q + kQB - 1) / kQB;
  const int tiles_per_block = (a.kv_stride + kKeys - 1) / kKeys;
  const long long total = static_cast<long long>(a.batch) * blocks_per_seq * tiles_per_block;
  auto kernel = a.fp8 ? sga_index_prefill_kernel<true> : sga_index_prefill_kernel<false>;
  const size_t smem = a.fp8 ? PrefillCfg<true>::kSmemBytes : PrefillCfg<false>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  PrefillParams p;
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.scores = a.scores;
  p.status = a.status;
  p.n_q = a.n_q;
  p.kv_stride = a.kv_stride;
  p.tiles_per_block = tiles_per_block;
  p.blocks_per_seq = blocks_per_seq;
  p.total_items = total;
  const int grid = static_cast<int>(total < num_sms ? total : num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(kPfThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, kmap, qmap, p);
}

}  // namespace

cudaError_t launch_index_scores(const IndexArgs& a, int num_sms, cudaStream_t stream) {
  const int rows = a.batch * a.n_q;
  const bool prefill = index_uses_prefill(a.n_q);
  // decode E4M3 tiles are 256 keys: one box of 256 rows
  const int tile_keys = (a.fp8 && !prefill) ? IndexCfg<true>::kTileKeys : kKeys;
  const int tiles_per_row = (a.kv_stride + tile_keys - 1) / tile_keys;
  const long long total = static_cast<long long>(rows) * tiles_per_row;
  if (total == 0) return cudaSuccess;
  const int esize = a.fp8 ? 1 : 2;
  const uint32_t strip = a.fp8 ? 128 : 64;  // elements per 128-byte strip
  CUtensorMap kmap, qmap;
  cudaError_t e = make_tmap_2d(&kmap, a.fp8, a.k_idx, kDim, static_cast<uint64_t>(a.batch) * a.kv_stride,
                               kDim * esize, strip, static_cast<uint32_t>(tile_keys));
  if (e != cudaSuccess) return e;
  e = make_tmap_2d(&qmap, a.fp8, a.q_idx, kDim, static_cast<uint64_t>(rows) * kHeads, kDim * esize, strip, kHeads);
  if (e != cudaSuccess) return e;
  if (prefill) return launch_prefill(a, num_sms, stream, kmap, qmap);
  const bool cand = a.cand != nullptr;
  if (cand && (a.hist == nullptr || a.cand_n == nullptr || a.kv_stride > kFusedTopkMaxL)) return cudaErrorInvalidValue;
  auto kernel = cand ? (a.fp8 ? sga_index_kernel<true, true> : sga_index_kernel<false, true>)
                     : (a.fp8 ? sga_index_kernel<true, false> : sga_index_kernel<false, false>);
  const size_t smem = a.fp8 ? IndexCfg<true>::kSmemBytes : IndexCfg<false>::kSmemBytes;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  IndexParams p;
  p.w = a.w;
  p.q_pos = a.q_pos;
  p.scores = a.scores;
  p.hist = a.hist;
  p.cand = a.cand;
  p.cand_n = a.cand_n;
  p.status = a.status;
  p.n_q = a.n_q;
  p.kv_stride = a.kv_stride;
  p.tiles_per_row = tiles_per_row;
  p.top_k = a.top_k;
  p.total_tiles = total;
  const int grid = static_cast<int>(total < num_sms ? total : num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(cand ? kCandThreads : kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, kmap, qmap, p);
}

}  // namespace sga
