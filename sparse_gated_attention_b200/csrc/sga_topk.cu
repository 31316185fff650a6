// Step 2: top-K selection (archdb "A.X K2", token-selection field: top-2048
// tokens per query; arXiv abstract "A.X K2 Technical Report": each query reads
// only 2,048 positions).  Larger score first; equal scores go to the lower
// position; output ascending, -1 padded.
//
// Scores are ranked through order_bits (an order-preserving 32-bit image of
// the float).  The K-th largest score key K* splits the positions into
// "above" (all selected) and "ties" (key == K*, of which the lowest positions
// fill the remaining slots); nothing else needs ordering.  One thread-block
// cluster of C CTAs (1024 threads each) handles one query; CTA r owns a
// contiguous segment of positions (a multiple of 128).
//
// Resident kernel (segments of at most 32768 positions, i.e. rows up to
// 8 x 32768): the whole segment is copied once into shared memory (eight
// 16-byte loads per thread, all in flight at once) and every pass reads it there.  Warp w owns 1024 consecutive
// positions of the segment and walks them 32 at a time, so a ballot over one
// step is the 32-position word of that step in position order.
//   1. MSD radix select over the score key, 12/12/8 bits per level: each CTA
//      counts its segment into a shared-memory histogram and all CTAs sum the
//      C histograms through distributed shared memory, so every CTA finds the
//      same bin.  Levels stop when that bin fits a candidate list (8192 keys)
//      or is a single key.  Under sga_forward the indexer has already counted
//      the first level, so that pass is skipped.
//   2. One ballot pass builds, per 32 positions, an "above" word (keys whose
//      bin lies above the selected bin: selected whatever K* is) and an
//      in-bin word; lane j keeps the words of step j.  If the bin is wider
//      than one key, its keys are listed in the CTA's candidate list (one
//      atomic per warp), each CTA pushes its list length to every CTA with a
//      remote store, and after one cluster barrier every CTA copies the other
//      lists over distributed shared memory and narrows them to K* itself (no
//      leader).
//   3. The in-bin bits are split against K* from the resident scores into
//      selected (key > K*) and tie (key == K*) bits.  Warp and block scans of
//      the word popcounts, plus the (selected, ties) counts every CTA pushes
//      to the others, give each set bit its output slot; ties are taken in
//      position order until the K slots are full.  Two cluster barriers follow
//      the radix levels and none precedes the exit.
// Streaming kernel (longer rows): the segment streams through a 3-slot ring of
// 32 KB bulk copies once per pass; the second step records selection / tie
// words (shared memory up to 65536 positions, else the workspace) and stages
// candidates per warp, own candidates are marked in the words after K* is
// known, and the words are emitted as above.
#include <cooperative_groups.h>

#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace cg = cooperative_groups;

namespace sga {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBits = kTopkHistBits;  // 12
constexpr int kBins = kTopkHistBins;  // 4096
constexpr int kBinsPerThread = kBins / kThreads;
constexpr int kCandCap = 8192;
constexpr int kMaxCluster = 8;
constexpr int kChunk = 8192;           // scores per ring slot (32 KB)
constexpr int kRingSlots = 3;
constexpr int kSegWordsSmem = 2048;    // bitmap words per segment kept in shared memory
constexpr int kMaxWordsPerThread = 8;  // bitmap words kept in registers per emission batch
constexpr size_t kRingBytes = kRingSlots * kChunk * 4;
constexpr int kWarpStage = 64;         // per-warp staging of candidates before one shared atomic
constexpr size_t kSmemBytes =
    kRingBytes + 2 * kBins * 4 + kCandCap * 8 + 2 * kSegWordsSmem * 4 + kWarps * kWarpStage * 8 + 4 * 8;
// resident kernel
constexpr int kResSeg = 32768;                  // positions per CTA held in shared memory (128 KB)
constexpr int kResWarpSpan = kResSeg / kWarps;  // 1024 consecutive positions per warp
constexpr int kResSteps = kResWarpSpan / 32;    // 32 ballot steps per warp and pass
constexpr size_t kResSmemBytes = kResSeg * 4 + 2 * kBins * 4 + kCandCap * 8;
static_assert(kResSteps == 32, "lane j keeps the words of step j");
static_assert(kSmemBytes + 2048 <= 232448 && kResSmemBytes + 2048 <= 232448, "shared memory budget");

struct TopkParams {
  const float* scores;
  const int32_t* q_pos;
  int32_t* idx;
  uint32_t* bitmap;
  uint32_t* hist;  // first-level histograms from the indexer (or null); zeroed here after use
  int* status;
  int kv_stride, top_k;
  long long words_per_row;
};

// ghist = the sum of every cluster CTA's lhist.  Thread t takes bins 4t .. 4t + 3:
// one 16-byte shared-memory load per CTA, four CTAs' loads issued before any
// is added.
__device__ __forceinline__ void cluster_hist_sum(cg::cluster_group& cluster, const uint32_t* lhist, uint32_t* ghist,
                                                 int C) {
  static_assert(kBins == 4 * kThreads, "four bins per thread");
  const int tid = threadIdx.x;
  constexpr int kInFlight = 4;
  uint4 acc = make_uint4(0u, 0u, 0u, 0u);
  for (int r0 = 0; r0 < C; r0 += kInFlight) {
    uint4 v[kInFlight];
#pragma unroll
    for (int k = 0; k < kInFlight; ++k)
      v[k] = r0 + k < C ? reinterpret_cast<const uint4*>(cluster.map_shared_rank(lhist, r0 + k))[tid]
                        : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < kInFlight; ++k) {
      acc.x += v[k].x;
      acc.y += v[k].y;
      acc.z += v[k].z;
      acc.w += v[k].w;
    }
  }
  reinterpret_cast<uint4*>(ghist)[tid] = acc;
}

// Inclusive block scan of one value per thread; also returns the block total.
__device__ __forceinline__ uint32_t block_inclusive_scan(uint32_t v, uint32_t* warp_buf, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_buf[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t x = warp_buf[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, x, o);
      if (lane >= o) x += u;
    }
    warp_buf[lane] = x;
  }
  __syncthreads();
  const uint32_t before = warp == 0 ? 0u : warp_buf[warp - 1];
  total = warp_buf[kWarps - 1];
  __syncthreads();
  return v + before;
}

struct Narrow {
  uint32_t digit, above, count;
};

// Finds the bin holding the `need`-th largest key: fewer than `need` keys lie
// in higher bins, at least `need` in this bin or higher.
__device__ __forceinline__ Narrow find_bin(const uint32_t* hist, uint32_t need, uint32_t* warp_buf, Narrow* out) {
  const int i = threadIdx.x;
  uint32_t h[kBinsPerThread];
  uint32_t sum = 0;
#pragma unroll
  for (int k = 0; k < kBinsPerThread; ++k) {
    h[k] = hist[kBins - 1 - (kBinsPerThread * i + k)];
    sum += h[k];
  }
  uint32_t total;
  const uint32_t incl = block_inclusive_scan(sum, warp_buf, total);
  uint32_t run = incl - sum;
  if (run < need && need <= incl) {
#pragma unroll
    for (int k = 0; k < kBinsPerThread; ++k) {
      if (run < need && need <= run + h[k]) {
        out->digit = kBins - 1 - (kBinsPerThread * i + k);
        out->above = run;
        out->count = h[k];
      }
      run += h[k];
    }
  }
  __syncthreads();
  return *out;
}

// Narrows the first nc candidates (key << 32 | ~position), all in the bin
// (prefix, mask, shift), to the exact K-th key with 8-bit radix levels: every
// thread counts into a 256-bin histogram in `ghist`, then one warp finds the
// bin with a warp scan (8 bins per lane) and publishes it, so a level costs
// three block barriers and no block-wide scan.  Every thread must call it after
// the list is complete.  Returns K* in the high 32 bits (kmask then covers all
// of them); `need` becomes the number of ties at K* still to take.
__device__ __noinline__ uint64_t refine_candidates(const uint64_t* cand, uint32_t nc, uint32_t* ghist, uint32_t prefix,
                                                   uint32_t mask, int shift, uint32_t& need, uint32_t* warp_buf,
                                                   Narrow* narrow, uint64_t& kmask) {
  (void)warp_buf;
  constexpr int kDigit = 8;
  const int tid = threadIdx.x, lane = tid & 31;
  kmask = static_cast<uint64_t>(mask) << 32;
  uint64_t kpref = static_cast<uint64_t>(prefix) << 32;
  while (shift > 0) {
    const int width = shift >= kDigit ? kDigit : shift;
    shift -= width;
    const int nbins = 1 << width;
    const uint32_t dmask = static_cast<uint32_t>(nbins - 1);
    if (tid < (1 << kDigit)) ghist[tid] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < nc; i += kThreads) {
      const uint64_t c = cand[i];
      if ((c & kmask) == kpref) atomicAdd(ghist + (static_cast<uint32_t>(c >> (32 + shift)) & dmask), 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l holds bins nbins-1-8l .. nbins-8-8l (descending keys)
      uint32_t h[8], sum = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int b = nbins - 1 - (8 * lane + k);
        h[k] = b >= 0 ? ghist[b] : 0u;
        sum += h[k];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - sum;
      if (excl < need && need <= incl) {  // exactly one lane
        uint32_t run = excl;
        bool found = false;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (!found && need <= run + h[k]) {
            narrow->digit = static_cast<uint32_t>(nbins - 1 - (8 * lane + k));
            narrow->above = run;
            found = true;
          }
          run += h[k];
        }
      }
    }
    __syncthreads();
    kpref |= static_cast<uint64_t>(narrow->digit) << (32 + shift);
    kmask |= static_cast<uint64_t>(dmask) << (32 + shift);
    need -= narrow->above;
  }
  __syncthreads();  // every thread has read `narrow` and the histogram before either is reused
  return kpref;
}

// Appends the other CTAs' candidate lists behind this CTA's `own` entries;
// peer_n[r] is the length of CTA r's list.  Returns the total length.  The
// caller's cluster barrier must have published every list and count, and no
// CTA may change the first entries of its list until all have copied them.
__device__ __forceinline__ uint32_t pull_candidates(cg::cluster_group& cluster, uint64_t* cand, uint32_t own,
                                                    const uint32_t* peer_n) {
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  uint32_t nc = own;
  for (int r = 0; r < C; ++r) {
    if (r == rank) continue;
    const uint32_t cnt = min(peer_n[r], static_cast<uint32_t>(kCandCap) - nc);
    const uint64_t* src = cluster.map_shared_rank(cand, r);
    for (uint32_t i = threadIdx.x; i < cnt; i += kThreads) cand[nc + i] = src[i];
    nc += cnt;
  }
  return nc;
}

// Streaming kernel: every CTA reads the other CTAs' list lengths, copies their
// lists behind its own `own` entries and narrows them to K* (see
// refine_candidates).  Ends with the list complete in every CTA; the caller's
// earlier cluster barrier must have published all lists.
__device__ __noinline__ void narrow_candidates(cg::cluster_group& cluster, uint64_t* cand, uint32_t* cand_n, uint32_t own,
                                               uint32_t* ghist, uint32_t prefix, uint32_t mask, int shift,
                                               uint32_t& need, uint32_t* warp_buf, Narrow* narrow, uint64_t& kpref,
                                               uint64_t& kmask) {
  uint32_t peer_n[kMaxCluster];
  const int C = static_cast<int>(cluster.num_blocks());
  for (int r = 0; r < C; ++r) peer_n[r] = *cluster.map_shared_rank(cand_n, r);
  const uint32_t nc = pull_candidates(cluster, cand, own, peer_n);
  cluster.sync();  // remote lists read; each CTA extended its own list behind its own entries
  kpref = refine_candidates(cand, nc, ghist, prefix, mask, shift, need, warp_buf, narrow, kmask);
}

// Four consecutive scores starting at s; positions >= end are read as 0 (the
// caller masks them).  The vector form needs rows that start 16-byte aligned.
template <bool kVec>
__device__ __forceinline__ float4 load4(const float* sc, int s, int end) {
  if (kVec) return __ldg(reinterpret_cast<const float4*>(sc + s));
  float4 v;
  v.x = s < end ? __ldg(sc + s) : 0.f;
  v.y = s + 1 < end ? __ldg(sc + s + 1) : 0.f;
  v.z = s + 2 < end ? __ldg(sc + s + 2) : 0.f;
  v.w = s + 3 < end ? __ldg(sc + s + 3) : 0.f;
  return v;
}

// Smallest / largest float whose order_bits lies in [lo_key, hi_key] (NaN bit
// patterns at the ends of the key range map to -inf / +inf).
__device__ __forceinline__ float key_to_float_lo(uint32_t k) {
  if (k <= 0x007FFFFFu) return -INFINITY;
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}
__device__ __forceinline__ float key_to_float_hi(uint32_t k) {
  if (k >= 0xFF800000u) return INFINITY;
  if (k == 0x7FFFFFFFu) k = 0x7FFFFFFEu;  // the key of -0.0: zeros fold onto +0.0, which lies above
  return __uint_as_float((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k);
}

// Merges a 4-bit nibble per lane into one 32-bit word per 8 lanes (lane 8w then
// holds the word for positions 32w .. 32w+31 of the warp's 128).
__device__ __forceinline__ uint32_t nibbles_to_word(uint32_t nib, int lane) {
  uint32_t w = nib << (4 * (lane & 7));
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 1);
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 2);
  w |= __shfl_xor_sync(0xFFFFFFFFu, w, 4);
  return w;
}

// Chunk j of the segment [s0, s1) into ring slot g % kRingSlots (bulk copy,
// completing on that slot's mbarrier); g counts chunks over all passes.
__device__ __forceinline__ void ring_issue(float* ring, uint32_t bar0, const float* sc, int s0, int s1, int g, int j) {
  const int slot = g % kRingSlots;
  const int pos = s0 + j * kChunk;
  const int cnt = min(kChunk, s1 - pos);
  const uint32_t bytes = static_cast<uint32_t>((cnt + 3) & ~3) * 4u;
  mbar_arrive_expect_tx(bar0 + 8u * slot, bytes);
  bulk_load(smem_u32(ring + slot * kChunk), sc + pos, bytes, bar0 + 8u * slot);
}

// Moves a warp's staged candidates to the CTA list with one shared atomic; returns 0.
__device__ __forceinline__ uint32_t flush_stage(uint32_t wcount, const uint64_t* wstage, uint64_t* cand,
                                                uint32_t* cand_n, int lane) {
  if (wcount == 0) return 0;
  __syncwarp();  // staged entries written by other lanes are visible
  uint32_t base = 0;
  if (lane == 0) base = atomicAdd(cand_n, wcount);
  base = __shfl_sync(0xFFFFFFFFu, base, 0);
  for (uint32_t i = lane; i < wcount; i += 32)
    if (base + i < kCandCap) cand[base + i] = wstage[i];
  __syncwarp();
  return 0;
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads, 1) sga_topk_stream_kernel(TopkParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  float* ring = reinterpret_cast<float*>(smem_raw);
  uint32_t* lhist = reinterpret_cast<uint32_t*>(smem_raw + kRingBytes);
  uint32_t* ghist = lhist + kBins;
  uint64_t* cand = reinterpret_cast<uint64_t*>(ghist + kBins);
  uint32_t* selw_s = reinterpret_cast<uint32_t*>(cand + kCandCap);
  uint32_t* tiew_s = selw_s + kSegWordsSmem;
  uint64_t* wstage = reinterpret_cast<uint64_t*>(tiew_s + kSegWordsSmem) + (threadIdx.x >> 5) * kWarpStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(tiew_s + kSegWordsSmem) + kWarps * kWarpStage;  // full[3], hist
  __shared__ uint32_t warp_buf[kWarps];
  __shared__ uint32_t warp_buf2[kWarps];
  __shared__ Narrow narrow;
  __shared__ uint32_t cand_n;     // candidates of this CTA's segment
  __shared__ uint32_t counts[2];  // this segment's (selected, ties), read by the whole cluster
  __shared__ int abort_flag;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31;
  const int K = p.top_k;
  int32_t* out = p.idx + static_cast<size_t>(row) * K;
  grid_dependency_wait();  // scores, histograms and q_pos come from earlier kernels
  grid_launch_dependents();
  uint32_t* hist_row = p.hist ? p.hist + static_cast<size_t>(row) * kBins : nullptr;
  const int t = __ldg(p.q_pos + row);
  if (t < 0 || t >= p.kv_stride) {
    if (rank == 0) {
      if (tid == 0) record_status(p.status, kStatusDeviceArg);
      for (int j = tid; j < K; j += kThreads) out[j] = -1;
      if (hist_row)
        for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
    }
    return;
  }
  const int n = t + 1;
  if (n <= K) {
    if (rank == 0) {
      for (int j = tid; j < K; j += kThreads) out[j] = j < n ? j : -1;
      if (hist_row)
        for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
    }
    return;
  }
  const float* sc = p.scores + static_cast<size_t>(row) * p.kv_stride;
  const int per = (((n + C - 1) / C) + 127) & ~127;
  const int s0 = min(rank * per, n), s1 = min(s0 + per, n);
  const int nch = (s1 - s0 + kChunk - 1) / kChunk;
  // selection / tie words of this segment: shared memory when they fit, else the workspace
  const int wbeg = s0 >> 5, wend = (s1 + 31) >> 5;
  const bool words_in_smem = wend - wbeg <= kSegWordsSmem;
  uint32_t* gsel = p.bitmap + static_cast<size_t>(row) * 2 * p.words_per_row;
  uint32_t* selw = words_in_smem ? selw_s : gsel;
  uint32_t* tiew = words_in_smem ? tiew_s : gsel + p.words_per_row;
  const int woff = words_in_smem ? wbeg : 0;
  const uint32_t bar0 = smem_u32(bars);
  const uint32_t hist_bar = bar0 + 8u * kRingSlots;
  if (tid == 0) {
    cand_n = 0;
    abort_flag = 0;
    for (int i = 0; i <= kRingSlots; ++i) mbar_init(bar0 + 8u * i, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (kVec && tid == 0) {
    if (p.hist) {
      mbar_arrive_expect_tx(hist_bar, kBins * 4);
      bulk_load(smem_u32(ghist), p.hist + static_cast<size_t>(row) * kBins, kBins * 4, hist_bar);
    }
    for (int j = 0; j < min(kRingSlots, nch); ++j) ring_issue(ring, bar0, sc, s0, s1, j, j);
  }
  int consumed = 0;  // ring chunks consumed by earlier passes (mbarrier phase bookkeeping)

  // ---- 1. radix levels on the score key until the bin fits the candidate list or is one key
  uint32_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(K);
  int shift = 32;
  uint32_t bucket = 0;
  bool first = true;
  while (true) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    if (first && p.hist) {
      if (kVec) {
        if (!mbar_wait(hist_bar, 0, &abort_flag)) record_status(p.status, kStatusTimeout);
      } else {
        for (int b = tid; b < kBins; b += kThreads) ghist[b] = hist_row[b];
      }
      __syncthreads();
    } else {
      for (int b = tid; b < kBins; b += kThreads) lhist[b] = 0;
      __syncthreads();
      if (kVec && consumed > 0 && tid == 0)
        for (int j = 0; j < min(kRingSlots, nch); ++j) ring_issue(ring, bar0, sc, s0, s1, consumed + j, j);
      for (int j = 0; j < nch; ++j) {
        const int g = consumed + j, slot = g % kRingSlots;
        if (kVec && !mbar_wait(bar0 + 8u * slot, static_cast<uint32_t>((g / kRingSlots) & 1), &abort_flag))
          record_status(p.status, kStatusTimeout);
        const int pos = s0 + j * kChunk, cnt = min(kChunk, s1 - pos);
        const float4* d4 = reinterpret_cast<const float4*>(ring + slot * kChunk);
        for (int f = tid; 4 * f < cnt; f += kThreads) {
          const int s = pos + 4 * f;
          const float4 v = kVec ? d4[f] : load4<false>(sc, s, s1);
          const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t k = order_bits(e[q]);
            if (s + q < s1 && (k & mask) == prefix) atomicAdd(lhist + ((k >> shift) & dmask), 1u);
          }
        }
        __syncthreads();  // slot fully read
        if (kVec && tid == 0 && j + kRingSlots < nch) ring_issue(ring, bar0, sc, s0, s1, g + kRingSlots, j + kRingSlots);
      }
      if (kVec) consumed += nch;
      cluster.sync();
      cluster_hist_sum(cluster, lhist, ghist, C);
      cluster.sync();  // every CTA has read every histogram
    }
    first = false;
    const Narrow nr = find_bin(ghist, need, warp_buf, &narrow);
    prefix |= nr.digit << shift;
    mask |= dmask << shift;
    need -= nr.above;
    bucket = nr.count;
    if (bucket <= kCandCap || shift == 0) break;
  }
  // A bin that is a single key holds exact ties: they go straight to the tie words.
  const bool resolved = shift == 0;

  // ---- 2. one pass over the segment: selection / tie words and local candidates.
  // The bin is the key range [prefix, prefix | ~mask]; as floats, "above" is
  // f > f_hi and "in the bin" is f_lo <= f <= f_hi, so most positions cost two
  // compares and warps with nothing to record skip the word assembly.
  const float f_lo = key_to_float_lo(prefix), f_hi = key_to_float_hi(prefix | ~mask);
  for (int w = wbeg + tid; w < wend; w += kThreads) {
    selw[w - woff] = 0u;
    tiew[w - woff] = 0u;
  }
  __syncthreads();
  uint32_t my_sel = 0, my_tie = 0;
  uint32_t wcount = 0;  // staged candidates of this warp (same value in every lane)
  if (kVec && consumed > 0 && tid == 0)
    for (int j = 0; j < min(kRingSlots, nch); ++j) ring_issue(ring, bar0, sc, s0, s1, consumed + j, j);
  for (int j = 0; j < nch; ++j) {
    const int g = consumed + j, slot = g % kRingSlots;
    if (kVec && !mbar_wait(bar0 + 8u * slot, static_cast<uint32_t>((g / kRingSlots) & 1), &abort_flag))
      record_status(p.status, kStatusTimeout);
    const int pos = s0 + j * kChunk, cnt = min(kChunk, s1 - pos);
    const float4* d4 = reinterpret_cast<const float4*>(ring + slot * kChunk);
    for (int f = tid; f < kChunk / 4; f += kThreads) {  // same trip count in every lane
      const int s = pos + 4 * f;
      float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      if (4 * f < cnt) v = kVec ? d4[f] : load4<false>(sc, s, s1);
      const float e[4] = {v.x, v.y, v.z, v.w};
      uint32_t nib_above = 0, nib_bin = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool valid = s + q < s1;
        nib_above |= static_cast<uint32_t>(valid && e[q] > f_hi) << q;
        nib_bin |= static_cast<uint32_t>(valid && e[q] >= f_lo && e[q] <= f_hi) << q;
      }
      if (!__any_sync(0xFFFFFFFFu, (nib_above | nib_bin) != 0)) continue;
      my_sel += __popc(nib_above);
      const uint32_t wa = nibbles_to_word(nib_above, lane);
      const uint32_t wb = nibbles_to_word(nib_bin, lane);
      if ((lane & 7) == 0 && s < s1) {
        if (wa) selw[(s >> 5) - woff] = wa;
        if (resolved && wb) tiew[(s >> 5) - woff] = wb;
      }
      if (resolved) {
        my_tie += __popc(nib_bin);
      } else if (__any_sync(0xFFFFFFFFu, nib_bin != 0)) {
        // stage this lane's in-bin keys in the warp's buffer: warp prefix of the per-lane counts
        const uint32_t c4 = __popc(nib_bin);
        uint32_t incl = c4;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (lane >= o) incl += y;
        }
        const uint32_t total = __shfl_sync(0xFFFFFFFFu, incl, 31);
        if (wcount + total > kWarpStage) wcount = flush_stage(wcount, wstage, cand, &cand_n, lane);
        if (total > kWarpStage) {  // more than a buffer in one step: straight to the list
          uint32_t base = 0;
          if (lane == 31) base = atomicAdd(&cand_n, total);
          base = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - c4;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if ((nib_bin >> q) & 1u) {
              if (base < kCandCap)
                cand[base] = (static_cast<uint64_t>(order_bits(e[q])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(s + q));
              ++base;
            }
          }
        } else {
          uint32_t off = wcount + incl - c4;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if ((nib_bin >> q) & 1u) {
              wstage[off] = (static_cast<uint64_t>(order_bits(e[q])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(s + q));
              ++off;
            }
          }
          wcount += total;
        }
      }
    }
    __syncthreads();  // slot fully read
    if (kVec && tid == 0 && j + kRingSlots < nch) ring_issue(ring, bar0, sc, s0, s1, g + kRingSlots, j + kRingSlots);
  }
  if (kVec) consumed += nch;
  if (!resolved) wcount = flush_stage(wcount, wstage, cand, &cand_n, lane);
  cluster.sync();  // segments scanned, candidate lists complete

  // ---- 3. every CTA: all candidates -> K*; mark own candidates; publish counts
  if (!resolved) {
    const uint32_t own = min(cand_n, static_cast<uint32_t>(kCandCap));
    uint64_t kpref, kmask;
    narrow_candidates(cluster, cand, &cand_n, own, ghist, prefix, mask, shift, need, warp_buf, &narrow, kpref, kmask);
    // own candidates (the first `own` entries) -> selection or tie bits in own words
    for (uint32_t i = tid; i < own; i += kThreads) {
      const uint64_t c = cand[i];
      const uint64_t hi = c & kmask;
      if (hi >= kpref) {
        const uint32_t s = 0xFFFFFFFFu - static_cast<uint32_t>(c);
        const bool tie = hi == kpref;
        atomicOr((tie ? tiew : selw) + ((s >> 5) - woff), 1u << (s & 31));
        if (tie) {
          ++my_tie;
        } else {
          ++my_sel;
        }
      }
    }
  }
  uint32_t seg_sel, seg_tie;
  block_inclusive_scan(my_sel, warp_buf, seg_sel);
  block_inclusive_scan(my_tie, warp_buf2, seg_tie);
  if (tid == 0) {
    counts[0] = seg_sel;
    counts[1] = seg_tie;
  }
  cluster.sync();  // counts published, own words marked
  uint32_t sel_before = 0, tie_before = 0, sel_all = 0, tie_all = 0;
  for (int r = 0; r < C; ++r) {
    const uint32_t* rc = cluster.map_shared_rank(counts, r);
    const uint32_t a = rc[0], b = rc[1];
    if (r < rank) {
      sel_before += a;
      tie_before += b;
    }
    sel_all += a;
    tie_all += b;
  }
  cluster.sync();  // every CTA has read every count (and its copy of the histogram row)
  if (rank == 0 && hist_row)  // ready for the next call
    for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
  const uint32_t take_all = static_cast<uint32_t>(K) > sel_all ? static_cast<uint32_t>(K) - sel_all : 0u;
  if (rank == 0 && tid == 0 &&
      (sel_all > static_cast<uint32_t>(K) || sel_all + tie_all < static_cast<uint32_t>(K)))
    record_status(p.status, kStatusDeviceArg);

  // ---- 4. emit this segment in position order
  uint32_t sel_run = sel_before, tie_run = tie_before;
  for (int wb = wbeg; wb < wend; wb += kThreads * kMaxWordsPerThread) {
    const int w0 = wb + tid * kMaxWordsPerThread;
    uint32_t sw[kMaxWordsPerThread], tw[kMaxWordsPerThread];
    uint32_t cs = 0, ct = 0;
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i) {
      const bool in = w0 + i < wend;
      sw[i] = in ? selw[w0 + i - woff] : 0u;
      tw[i] = in ? tiew[w0 + i - woff] : 0u;
      cs += __popc(sw[i]);
      ct += __popc(tw[i]);
    }
    uint32_t bs, bt;
    const uint32_t s_incl = block_inclusive_scan(cs, warp_buf, bs);
    const uint32_t t_incl = block_inclusive_scan(ct, warp_buf2, bt);
    const uint32_t tb = tie_run + t_incl - ct;
    uint32_t pos = sel_run + (s_incl - cs) + min(tb, take_all);
    uint32_t ties_left = tb < take_all ? take_all - tb : 0u;
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i) {
      uint32_t t2 = tw[i], keep = 0;
      while (t2 && ties_left) {
        const uint32_t low = t2 & (0u - t2);
        keep |= low;
        t2 ^= low;
        --ties_left;
      }
      uint32_t mm = sw[i] | keep;
      while (mm) {
        const int b = __ffs(mm) - 1;
        mm &= mm - 1;
        if (pos < static_cast<uint32_t>(K)) out[pos] = (w0 + i) * 32 + b;
        ++pos;
      }
    }
    sel_run += bs;
    tie_run += bt;
  }
  if (rank == 0) {
    const uint32_t emitted = sel_all + min(tie_all, take_all);
    for (int j = static_cast<int>(emitted) + tid; j < K; j += kThreads) out[j] = -1;
  }
}

template <bool kVec>
__global__ void __launch_bounds__(kThreads, 1) sga_topk_resident_kernel(TopkParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  float* seg = reinterpret_cast<float*>(smem_raw);
  uint32_t* lhist = reinterpret_cast<uint32_t*>(smem_raw + kResSeg * 4);
  uint32_t* ghist = lhist + kBins;
  uint64_t* cand = reinterpret_cast<uint64_t*>(ghist + kBins);
  __shared__ uint32_t warp_buf[kWarps];
  __shared__ uint32_t wsel[kWarps], wtie[kWarps];  // per-warp exclusive prefixes of the word popcounts
  __shared__ Narrow narrow;
  __shared__ uint32_t cand_n;
  __shared__ uint32_t peer_n[kMaxCluster];          // candidate-list lengths, written by each CTA of the cluster
  __shared__ uint32_t peer_counts[kMaxCluster][2];  // (selected, ties) of each CTA's segment, written by that CTA

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.top_k;
  int32_t* out = p.idx + static_cast<size_t>(row) * K;
  grid_dependency_wait();  // scores, histograms and q_pos come from earlier kernels
  grid_launch_dependents();
  uint32_t* hist_row = p.hist ? p.hist + static_cast<size_t>(row) * kBins : nullptr;
  const int t = __ldg(p.q_pos + row);
  if (t < 0 || t >= p.kv_stride) {
    if (rank == 0) {
      if (tid == 0) record_status(p.status, kStatusDeviceArg);
      for (int j = tid; j < K; j += kThreads) out[j] = -1;
      if (hist_row)
        for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
    }
    return;
  }
  const int n = t + 1;
  if (n <= K) {
    if (rank == 0) {
      for (int j = tid; j < K; j += kThreads) out[j] = j < n ? j : -1;
      if (hist_row)
        for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
    }
    return;
  }
  // The host picks C with C * kResSeg >= kv_stride, so every segment fits.
  const float* sc = p.scores + static_cast<size_t>(row) * p.kv_stride;
  const int per = (((n + C - 1) / C) + 127) & ~127;
  const int s0 = min(rank * per, n), s1 = min(s0 + per, n);
  const int len = s1 - s0;
  if (tid == 0) cand_n = 0;
  if (kVec) {
    // The whole segment with 16-byte loads from every thread, all in flight at
    // once (rows are 16-byte aligned and kv_stride % 4 == 0, so rounding the
    // length up to 4 stays inside the row), and the histogram row likewise.
    constexpr int kPerThread = kResSeg / 4 / kThreads;  // 8 float4
    const float4* src = reinterpret_cast<const float4*>(sc + s0);
    const int n4 = (len + 3) >> 2;
    float4 v[kPerThread];
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = tid + k * kThreads;
      if (i < n4) v[k] = __ldcg(src + i);
    }
    uint4 hv = make_uint4(0u, 0u, 0u, 0u);
    if (p.hist) hv = __ldcg(reinterpret_cast<const uint4*>(hist_row) + tid);
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = tid + k * kThreads;
      if (i < n4) reinterpret_cast<float4*>(seg)[i] = v[k];
    }
    if (p.hist) reinterpret_cast<uint4*>(ghist)[tid] = hv;
  } else {
    for (int i = tid; i < len; i += kThreads) seg[i] = __ldg(sc + s0 + i);
    if (p.hist) {
      for (int b = tid; b < kBins; b += kThreads) ghist[b] = hist_row[b];
    }
  }
  __syncthreads();
  static_assert(kBins == 4 * kThreads, "one uint4 of the histogram row per thread");
  const int wbase = warp * kResWarpSpan;  // this warp's first position within the segment

  // ---- 1. radix levels on the score key until the bin fits the candidate list or is one key
  uint32_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(K);
  int shift = 32;
  uint32_t bucket = 0;
  bool first = true;
  while (true) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    if (first && p.hist) {
      // the first level comes from the indexer's histogram, already in ghist
    } else {
      for (int b = tid; b < kBins; b += kThreads) lhist[b] = 0;
      __syncthreads();
#pragma unroll 4
      for (int j = 0; j < kResSteps; ++j) {
        const int i = wbase + 32 * j + lane;
        if (i < len) {
          const uint32_t k = order_bits(seg[i]);
          if ((k & mask) == prefix) atomicAdd(lhist + ((k >> shift) & dmask), 1u);
        }
      }
      cluster.sync();
      cluster_hist_sum(cluster, lhist, ghist, C);
      cluster.sync();  // every CTA has read every histogram
    }
    first = false;
    const Narrow nr = find_bin(ghist, need, warp_buf, &narrow);
    prefix |= nr.digit << shift;
    mask |= dmask << shift;
    need -= nr.above;
    bucket = nr.count;
    if (bucket <= kCandCap || shift == 0) break;
  }
  const bool resolved = shift == 0;  // the bin is a single key: its positions are the ties

  // ---- 2. one pass: per 32 positions a word of keys above the bin and a word
  // of keys in it (lane j keeps the words of step j).  As floats, "above" is
  // f > f_hi and "in the bin" f_lo <= f <= f_hi.
  const float f_lo = key_to_float_lo(prefix), f_hi = key_to_float_hi(prefix | ~mask);
  uint32_t my_sel = 0, my_bin = 0;
#pragma unroll 8
  for (int j = 0; j < kResSteps; ++j) {
    const int i = wbase + 32 * j + lane;
    const float f = i < len ? seg[i] : f_lo;
    const uint32_t sw = __ballot_sync(0xFFFFFFFFu, i < len && f > f_hi);
    const uint32_t bw = __ballot_sync(0xFFFFFFFFu, i < len && f >= f_lo && f <= f_hi);
    if (lane == j) {
      my_sel = sw;
      my_bin = bw;
    }
  }
  const int lpos = wbase + 32 * lane;  // segment offset of bit 0 of this lane's words
  uint32_t kstar = prefix;
  uint32_t my_tie = my_bin;
  if (!resolved) {
    // in-bin keys -> this CTA's candidate list (one shared atomic per warp)
    const uint32_t c = __popc(my_bin);
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += y;
    }
    uint32_t base = 0;
    if (lane == 31 && incl) base = atomicAdd(&cand_n, incl);
    base = __shfl_sync(0xFFFFFFFFu, base, 31) + incl - c;
    for (uint32_t m = my_bin; m; m &= m - 1, ++base) {
      const int i = lpos + __ffs(m) - 1;
      if (base < kCandCap)
        cand[base] = (static_cast<uint64_t>(order_bits(seg[i])) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(s0 + i));
    }
    __syncthreads();  // this CTA's list is complete
    if (tid < C) *cluster.map_shared_rank(&peer_n[rank], tid) = min(cand_n, static_cast<uint32_t>(kCandCap));
    cluster.sync();  // every list and every length published
    const uint32_t nc = pull_candidates(cluster, cand, peer_n[rank], peer_n);
    __syncthreads();  // the whole cluster's candidates are in this CTA's list
    uint64_t kmask;
    kstar = static_cast<uint32_t>(refine_candidates(cand, nc, ghist, prefix, mask, shift, need, warp_buf, &narrow,
                                                    kmask) >> 32);
    // in-bin positions: above K* -> selected, at K* -> ties, below -> dropped
    my_tie = 0;
    for (uint32_t m = my_bin; m; m &= m - 1) {
      const int b = __ffs(m) - 1;
      const uint32_t k = order_bits(seg[lpos + b]);
      if (k > kstar) my_sel |= 1u << b;
      if (k == kstar) my_tie |= 1u << b;
    }
  }

  // ---- 3. counts, their scans across warps and CTAs, emission in position order
  const uint32_t cs = __popc(my_sel), ct = __popc(my_tie);
  uint32_t is = cs, it = ct;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t ys = __shfl_up_sync(0xFFFFFFFFu, is, o);
    const uint32_t yt = __shfl_up_sync(0xFFFFFFFFu, it, o);
    if (lane >= o) {
      is += ys;
      it += yt;
    }
  }
  if (lane == 31) {
    wsel[warp] = is;
    wtie[warp] = it;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t xs = wsel[lane], xt = wtie[lane];
    uint32_t ps = xs, pt = xt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t ys = __shfl_up_sync(0xFFFFFFFFu, ps, o);
      const uint32_t yt = __shfl_up_sync(0xFFFFFFFFu, pt, o);
      if (lane >= o) {
        ps += ys;
        pt += yt;
      }
    }
    wsel[lane] = ps - xs;
    wtie[lane] = pt - xt;
    const uint32_t tot_s = __shfl_sync(0xFFFFFFFFu, ps, 31), tot_t = __shfl_sync(0xFFFFFFFFu, pt, 31);
    if (lane < C) {
      uint32_t* dst = cluster.map_shared_rank(&peer_counts[rank][0], lane);
      dst[0] = tot_s;
      dst[1] = tot_t;
    }
  }
  // Every count delivered (and every CTA's copy of the histogram row taken).
  // No CTA touches another's shared memory after this barrier, so none has to
  // wait for the others before exiting.
  cluster.sync();
  if (rank == 0 && hist_row)  // ready for the next call
    for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
  uint32_t sel_before = 0, tie_before = 0, sel_all = 0, tie_all = 0;
  for (int r = 0; r < C; ++r) {
    const uint32_t a = peer_counts[r][0], b = peer_counts[r][1];
    if (r < rank) {
      sel_before += a;
      tie_before += b;
    }
    sel_all += a;
    tie_all += b;
  }
  if (rank == 0 && tid == 0 && (sel_all + need != static_cast<uint32_t>(K) || tie_all < need))
    record_status(p.status, kStatusDeviceArg);
  SGA_DCHECK(p.status, resolved || cand_n <= static_cast<uint32_t>(kCandCap));  // the bin fit the candidate list
  const uint32_t sel_base = sel_before + wsel[warp] + (is - cs);
  const uint32_t tie_base = tie_before + wtie[warp] + (it - ct);
  const int pos0 = s0 + lpos;
  for (uint32_t m = my_sel | my_tie; m; m &= m - 1) {
    const int b = __ffs(m) - 1;
    const uint32_t below = (1u << b) - 1u;
    const uint32_t tr = tie_base + __popc(my_tie & below);
    if (((my_tie >> b) & 1u) && tr >= need) continue;
    const uint32_t slot = sel_base + __popc(my_sel & below) + min(tr, need);
    SGA_DCHECK(p.status, slot < static_cast<uint32_t>(K) && pos0 + b <= t);
    if (slot < static_cast<uint32_t>(K)) out[slot] = pos0 + b;
  }
  if (rank == 0) {
    const uint32_t emitted = sel_all + min(tie_all, need);
    for (int j = static_cast<int>(emitted) + tid; j < K; j += kThreads) out[j] = -1;
  }
}


// ---- selection from the indexer's candidates
// One CTA per row.  The indexer kept every key of the row that can still be
// among its top K, with its position, and counted the first radix level of
// those keys, which is exact at and above the K-th key's bin, so that bin
// comes from the histogram.  While the bin holds more keys than the list
// takes, further levels narrow it with passes over the candidates.  Then one
// pass marks the candidates above the bin in a position bitmap and lists the
// ones inside it; the list is refined to the exact K-th key K*, its keys above
// K* join the bitmap and its keys equal to K* form a tie bitmap, and both are
// emitted in position order, the lowest positions first among the ties.
constexpr int kFMaxWords = kFusedTopkMaxL / 32;
constexpr int kFWordsPerThread = kFMaxWords / kThreads;
constexpr int kFBatch = 8;  // candidate loads in flight per thread
constexpr int kFListCap = 8192;  // keys of the K-th key's bin listed without a further level
constexpr size_t kFSmemBytes = 2 * kFMaxWords * 4 + kBins * 4 + kFListCap * 8;
static_assert(kFMaxWords % kThreads == 0, "whole bitmap words per thread");

struct TopkCandParams {
  const uint64_t* cand;
  uint32_t* cand_n;
  uint32_t* hist;
  const int32_t* q_pos;
  int32_t* idx;
  int* status;
  int kv_stride, top_k;
};

__global__ void __launch_bounds__(kThreads, 1) sga_topk_cand_kernel(TopkCandParams p) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint32_t* selw = reinterpret_cast<uint32_t*>(smem_raw);        // [kFMaxWords] selected positions
  uint32_t* tiew = selw + kFMaxWords;                             // [kFMaxWords] positions of keys equal to K*
  uint32_t* ghist = tiew + kFMaxWords;                            // [kBins]
  uint64_t* list = reinterpret_cast<uint64_t*>(ghist + kBins);   // [kFListCap] the K-th key's bin
  __shared__ uint32_t warp_buf[kWarps], warp_buf2[kWarps];
  __shared__ Narrow narrow;
  __shared__ uint32_t list_n;

  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31;
  const int K = p.top_k;
  int32_t* out = p.idx + static_cast<size_t>(row) * K;
  grid_dependency_wait();  // candidates, counts and histograms come from the indexer
  grid_launch_dependents();
  uint32_t* hist_row = p.hist + static_cast<size_t>(row) * kBins;
  const int t = __ldg(p.q_pos + row);
  const bool bad = t < 0 || t >= p.kv_stride;
  const int n = bad ? 0 : t + 1;
  uint32_t nc = __ldcg(p.cand_n + static_cast<size_t>(row) * kCandNStride);
  __syncthreads();  // every thread has read the count before it is cleared for the next call
  if (tid == 0) p.cand_n[static_cast<size_t>(row) * kCandNStride] = 0u;
  SGA_DCHECK(p.status, nc <= static_cast<uint32_t>(n));
  nc = min(nc, static_cast<uint32_t>(n));
  if (bad || n <= K) {
    if (bad && tid == 0) record_status(p.status, kStatusDeviceArg);
    for (int j = tid; j < K; j += kThreads) out[j] = j < n ? j : -1;
    for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;
    return;
  }
  const int words = (n + 31) >> 5;
  reinterpret_cast<uint4*>(ghist)[tid] = __ldcg(reinterpret_cast<const uint4*>(hist_row) + tid);
  for (int w = tid; w < words; w += kThreads) {
    selw[w] = 0u;
    tiew[w] = 0u;
  }
  if (tid == 0) list_n = 0u;
  __syncthreads();
  for (int b = tid; b < kBins; b += kThreads) hist_row[b] = 0;  // read above; ready for the next call

  const uint64_t* cr = p.cand + static_cast<size_t>(row) * p.kv_stride;
  const Narrow nr = find_bin(ghist, static_cast<uint32_t>(K), warp_buf, &narrow);
  uint32_t prefix = nr.digit << (32 - kBits);
  uint32_t mask = ~((1u << (32 - kBits)) - 1u);
  uint32_t need = static_cast<uint32_t>(K) - nr.above;
  uint32_t count = nr.count;
  int shift = 32 - kBits;
  // ---- 1. while the bin holds more keys than the list takes: one more level
  // over the candidates (every key of the bin is a candidate)
  while (count > static_cast<uint32_t>(kFListCap) && shift > 0) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += kThreads) ghist[b] = 0;
    __syncthreads();
    for (uint32_t i0 = 0; i0 < nc; i0 += kFBatch * kThreads) {
      uint32_t kk[kFBatch];
#pragma unroll
      for (int u = 0; u < kFBatch; ++u) {
        const uint32_t i = i0 + u * kThreads + tid;
        kk[u] = i < nc ? static_cast<uint32_t>(__ldcg(cr + i) >> 32) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kFBatch; ++u)
        if (i0 + u * kThreads + tid < nc && (kk[u] & mask) == prefix)
          atomicAdd(ghist + ((kk[u] >> shift) & dmask), 1u);
    }
    __syncthreads();
    const Narrow nb = find_bin(ghist, need, warp_buf, &narrow);
    prefix |= nb.digit << shift;
    mask |= dmask << shift;
    need -= nb.above;
    count = nb.count;
  }
  // ---- 2. one pass: keys above the bin join the bitmap, keys inside it are
  // listed (or, once all 32 bits are fixed, are the ties themselves)
  const bool listing = shift > 0;
  for (uint32_t i0 = 0; i0 < nc; i0 += kFBatch * kThreads) {
    uint64_t cb[kFBatch];
#pragma unroll
    for (int u = 0; u < kFBatch; ++u) {
      const uint32_t i = i0 + u * kThreads + tid;
      cb[u] = i < nc ? __ldcg(cr + i) : 0ull;
    }
    uint32_t inm = 0;  // which of this thread's batch entries lie in the bin
#pragma unroll
    for (int u = 0; u < kFBatch; ++u) {
      const uint32_t k = static_cast<uint32_t>(cb[u] >> 32), pos = static_cast<uint32_t>(cb[u]);
      const bool valid = i0 + u * kThreads + tid < nc && pos <= static_cast<uint32_t>(t);
      SGA_DCHECK(p.status, i0 + u * kThreads + tid >= nc || pos <= static_cast<uint32_t>(t));
      const bool in = valid && (k & mask) == prefix;
      if (valid && (k & mask) > prefix) atomicOr(selw + (pos >> 5), 1u << (pos & 31));
      if (in && !listing) atomicOr(tiew + (pos >> 5), 1u << (pos & 31));
      inm |= static_cast<uint32_t>(in) << u;
    }
    if (listing) {
      // one list update per warp and batch: a warp scan of the lanes' counts
      const uint32_t cnt = static_cast<uint32_t>(__popc(inm));
      uint32_t incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
      }
      uint32_t base = 0;
      const uint32_t wtotal = __shfl_sync(0xFFFFFFFFu, incl, 31);
      if (lane == 0 && wtotal != 0u) base = atomicAdd(&list_n, wtotal);
      uint32_t slot = __shfl_sync(0xFFFFFFFFu, base, 0) + incl - cnt;
#pragma unroll
      for (int u = 0; u < kFBatch; ++u) {
        if ((inm >> u) & 1u) {
          SGA_DCHECK(p.status, slot < static_cast<uint32_t>(kFListCap));
          if (slot < static_cast<uint32_t>(kFListCap)) list[slot] = cb[u];
          ++slot;
        }
      }
    }
  }
  __syncthreads();  // bitmap and list complete
  // ---- 3. the exact K-th key K*, and the listed keys split against it
  if (listing) {
    const uint32_t ln = min(list_n, static_cast<uint32_t>(kFListCap));
    SGA_DCHECK(p.status, ln == count);
    uint64_t kmask;
    const uint32_t kstar = static_cast<uint32_t>(
        refine_candidates(list, ln, ghist, prefix, mask, shift, need, warp_buf, &narrow, kmask) >> 32);
    for (uint32_t i = tid; i < ln; i += kThreads) {
      const uint64_t c = list[i];
      const uint32_t k = static_cast<uint32_t>(c >> 32), pos = static_cast<uint32_t>(c);
      if (k > kstar) atomicOr(selw + (pos >> 5), 1u << (pos & 31));
      if (k == kstar) atomicOr(tiew + (pos >> 5), 1u << (pos & 31));
    }
    __syncthreads();
  }
  // ---- 4. emission in position order: the selected words plus the first `need` ties
  const int w0 = tid * kFWordsPerThread;
  uint32_t sw[kFWordsPerThread], tw[kFWordsPerThread];
  uint32_t cs = 0, ct = 0;
#pragma unroll
  for (int i = 0; i < kFWordsPerThread; ++i) {
    const bool inw = w0 + i < words;
    sw[i] = inw ? selw[w0 + i] : 0u;
    tw[i] = inw ? tiew[w0 + i] : 0u;
    cs += __popc(sw[i]);
    ct += __popc(tw[i]);
  }
  uint32_t sel_all, tie_all;
  const uint32_t s_incl = block_inclusive_scan(cs, warp_buf, sel_all);
  const uint32_t t_incl = block_inclusive_scan(ct, warp_buf2, tie_all);
  SGA_DCHECK(p.status, sel_all + need == static_cast<uint32_t>(K) && tie_all >= need);
  const uint32_t tb = t_incl - ct;  // ties in the words of lower threads
  uint32_t pos = (s_incl - cs) + min(tb, need);
  uint32_t ties_left = tb < need ? need - tb : 0u;
#pragma unroll
  for (int i = 0; i < kFWordsPerThread; ++i) {
    uint32_t t2 = tw[i], keep = 0;
    while (t2 && ties_left) {
      const uint32_t low = t2 & (0u - t2);
      keep |= low;
      t2 ^= low;
      --ties_left;
    }
    for (uint32_t m = sw[i] | keep; m; m &= m - 1) {
      const int b = __ffs(m) - 1;
      if (pos < static_cast<uint32_t>(K)) out[pos] = (w0 + i) * 32 + b;
      ++pos;
    }
  }
  const uint32_t emitted = min(sel_all + min(tie_all, need), static_cast<uint32_t>(K));
  for (int j = static_cast<int>(emitted) + tid; j < K; j += kThreads) out[j] = -1;
}

}  // namespace

// Words of one bitmap per row; the workspace holds two per row (selected, ties).
size_t topk_bitmap_words(int kv_stride) { return (static_cast<size_t>(kv_stride) + 31) / 32; }

// CTAs per query: enough to fill the GPU once, at most kMaxCluster.
int topk_cluster_size(int rows) {
  int c = 1;
  while (c < kMaxCluster && static_cast<long long>(rows) * c * 2 <= 148) c *= 2;
  return c;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  const bool vec = (a.kv_stride % 4 == 0) && (reinterpret_cast<uintptr_t>(a.scores) % 16 == 0);
  // rows that fit kMaxCluster segments of kResSeg positions take the resident kernel
  const int c_res = (a.kv_stride + kResSeg - 1) / kResSeg;
  const bool resident = c_res <= kMaxCluster;
  auto kernel = resident ? (vec ? sga_topk_resident_kernel<true> : sga_topk_resident_kernel<false>)
                         : (vec ? sga_topk_stream_kernel<true> : sga_topk_stream_kernel<false>);
  const size_t smem = resident ? kResSmemBytes : kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  TopkParams p;
  p.scores = a.scores;
  p.q_pos = a.q_pos;
  p.idx = a.idx;
  p.bitmap = a.bitmap;
  p.hist = a.hist;
  p.status = a.status;
  p.kv_stride = a.kv_stride;
  p.top_k = a.top_k;
  p.words_per_row = static_cast<long long>(topk_bitmap_words(a.kv_stride));
  int C = topk_cluster_size(a.rows);
  if (resident) C = max(C, c_res);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.rows * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

cudaError_t launch_topk_candidates(const TopkCandArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  if (a.kv_stride > kFusedTopkMaxL) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sga_topk_cand_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kFSmemBytes));
  if (e != cudaSuccess) return e;
  TopkCandParams p;
  p.cand = a.cand;
  p.cand_n = a.cand_n;
  p.hist = a.hist;
  p.q_pos = a.q_pos;
  p.idx = a.idx;
  p.status = a.status;
  p.kv_stride = a.kv_stride;
  p.top_k = a.top_k;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.rows));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kFSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sga_topk_cand_kernel, p);
}

}  // namespace sga
