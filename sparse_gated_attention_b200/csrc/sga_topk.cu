// Step 2: top-K selection (archdb "A.X K2", token-selection field: top-2048
// tokens per query; arXiv abstract "A.X K2 Technical Report": each query reads
// only 2,048 positions).  Larger score first; equal scores go to the lower
// position; output ascending, -1 padded.
//
// Each candidate s gets a unique 64-bit key
//     order_bits(score[s]) << 32  |  (0xFFFFFFFF - s)
// so "larger key" is exactly the selection order and the K-th largest key is a
// single threshold.  One thread-block cluster of C CTAs (1024 threads each)
// handles one query; CTA r owns a contiguous segment of the positions.
//   1. MSD radix select over the keys, 12 bits per level.  Each CTA counts its
//      segment into a shared-memory histogram; every CTA then sums the C
//      histograms through distributed shared memory, so all agree on the bin
//      that holds the threshold.  Levels stop once that bin fits the leader's
//      candidate list (8192 keys).  When the indexer has already counted the
//      first level (sga_forward) that pass is skipped.
//   2. One pass over the segments: a selection bitmap word per 32 positions
//      (warp ballot) marks keys above the bin; keys inside the bin are appended
//      to the leader CTA's candidate list through distributed shared memory.
//   3. The leader finishes the select among the candidates in shared memory,
//      sets their bitmap bits, and emits the set bits in position order
//      (per-thread popcounts + block scan).
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
constexpr int kUnroll = 4;
constexpr size_t kSmemBytes = 2 * kBins * 4 + kCandCap * 8;

struct TopkParams {
  const float* scores;
  const int32_t* q_pos;
  int32_t* idx;
  uint32_t* bitmap;
  const uint32_t* hist;
  int* status;
  int kv_stride, top_k;
  long long words_per_row;
};

__device__ __forceinline__ uint64_t sel_key(float f, int s) {
  return (static_cast<uint64_t>(order_bits(f)) << 32) | static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(s));
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
// in higher bins, at least `need` in this bin or higher.  Bins only up to
// `nbins` are used (the last level can be narrower than 12 bits).
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

__global__ void __launch_bounds__(kThreads, 1) sga_topk_kernel(TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* lhist = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* ghist = lhist + kBins;
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw + 2 * kBins * 4);
  __shared__ uint32_t warp_buf[kWarps];
  __shared__ Narrow narrow;
  __shared__ uint32_t cand_n;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  const int row = blockIdx.x / C;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.top_k;
  int32_t* out = p.idx + static_cast<size_t>(row) * K;
  const int t = __ldg(p.q_pos + row);
  if (t < 0 || t >= p.kv_stride) {
    if (rank == 0) {
      if (tid == 0) record_status(p.status, kStatusDeviceArg);
      for (int j = tid; j < K; j += kThreads) out[j] = -1;
    }
    return;
  }
  const int n = t + 1;
  if (n <= K) {
    if (rank == 0)
      for (int j = tid; j < K; j += kThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* sc = p.scores + static_cast<size_t>(row) * p.kv_stride;
  uint32_t* bits = p.bitmap + static_cast<size_t>(row) * p.words_per_row;
  const int per = (((n + C - 1) / C) + 31) & ~31;
  const int s0 = min(rank * per, n), s1 = min(s0 + per, n);
  if (tid == 0) cand_n = 0;

  // ---- 1. radix levels until the threshold bin fits the candidate list
  uint64_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(K);
  int shift = 64;
  uint32_t bucket = 0;
  bool first = true;
  while (true) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    if (first && p.hist) {
      const uint32_t* hrow = p.hist + static_cast<size_t>(row) * kBins;
      for (int b = tid; b < kBins; b += kThreads) ghist[b] = __ldg(hrow + b);
      __syncthreads();
    } else {
      for (int b = tid; b < kBins; b += kThreads) lhist[b] = 0;
      __syncthreads();
      for (int base = s0; base < s1; base += kUnroll * kThreads) {
        float v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int s = base + u * kThreads + tid;
          v[u] = s < s1 ? __ldg(sc + s) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int s = base + u * kThreads + tid;
          if (s < s1) {
            const uint64_t c = sel_key(v[u], s);
            if ((c & mask) == prefix) atomicAdd(lhist + (static_cast<uint32_t>(c >> shift) & dmask), 1u);
          }
        }
      }
      cluster.sync();
      for (int b = tid; b < kBins; b += kThreads) {
        uint32_t acc = 0;
        for (int r = 0; r < C; ++r) acc += cluster.map_shared_rank(lhist, r)[b];
        ghist[b] = acc;
      }
      cluster.sync();  // every CTA has read every histogram
    }
    first = false;
    const Narrow nr = find_bin(ghist, need, warp_buf, &narrow);
    prefix |= static_cast<uint64_t>(nr.digit) << shift;
    mask |= static_cast<uint64_t>(dmask) << shift;
    need -= nr.above;
    bucket = nr.count;
    if (bucket <= kCandCap || shift == 0) break;
  }

  // ---- 2. bitmap of keys above the bin; keys in the bin -> leader's candidate list
  cluster.sync();  // the leader's cand_n is initialised
  uint64_t* lead_cand = cluster.map_shared_rank(cand, 0);
  uint32_t* lead_n = cluster.map_shared_rank(&cand_n, 0);
  for (int base = s0; base < s1; base += kUnroll * kThreads) {
    float v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + u * kThreads + tid;
      v[u] = s < s1 ? __ldg(sc + s) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int s = base + u * kThreads + tid;
      bool above = false, in_bin = false;
      uint64_t c = 0;
      if (s < s1) {
        c = sel_key(v[u], s);
        above = (c & mask) > prefix;
        in_bin = (c & mask) == prefix;
      }
      const uint32_t word = __ballot_sync(0xFFFFFFFFu, above);
      const int first_pos = base + u * kThreads + warp * 32;
      if (lane == 0 && first_pos < s1) bits[first_pos >> 5] = word;
      const uint32_t cm = __ballot_sync(0xFFFFFFFFu, in_bin);
      if (cm) {
        uint32_t off = 0;
        if (lane == 0) off = atomicAdd(lead_n, static_cast<uint32_t>(__popc(cm)));
        off = __shfl_sync(0xFFFFFFFFu, off, 0);
        if (in_bin) {
          const uint32_t r = off + __popc(cm & ((1u << lane) - 1u));
          if (r < kCandCap) lead_cand[r] = c;
        }
      }
    }
  }
  cluster.sync();  // all candidates appended, all bitmap words written
  if (rank != 0) return;

  // ---- 3. leader: finish the select inside the candidate list
  const uint32_t nc = cand_n < kCandCap ? cand_n : kCandCap;
  while (need < bucket && shift > 0) {
    const int width = shift >= kBits ? kBits : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += kThreads) ghist[b] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < nc; i += kThreads) {
      const uint64_t c = cand[i];
      if ((c & mask) == prefix) atomicAdd(ghist + (static_cast<uint32_t>(c >> shift) & dmask), 1u);
    }
    __syncthreads();
    const Narrow nr = find_bin(ghist, need, warp_buf, &narrow);
    prefix |= static_cast<uint64_t>(nr.digit) << shift;
    mask |= static_cast<uint64_t>(dmask) << shift;
    need -= nr.above;
    bucket = nr.count;
  }
  for (uint32_t i = tid; i < nc; i += kThreads) {
    const uint64_t c = cand[i];
    if ((c & mask) >= prefix) {
      const uint32_t s = 0xFFFFFFFFu - static_cast<uint32_t>(c);
      atomicOr(bits + (s >> 5), 1u << (s & 31));
    }
  }
  __syncthreads();

  // ---- emit set bits in position order
  const int words = (n + 31) >> 5;
  const int per_t = (words + kThreads - 1) / kThreads;
  const int w0 = min(tid * per_t, words), w1 = min(w0 + per_t, words);
  uint32_t cnt = 0;
  for (int wi = w0; wi < w1; ++wi) cnt += __popc(__ldcg(bits + wi));
  uint32_t total;
  uint32_t pos = block_inclusive_scan(cnt, warp_buf, total) - cnt;
  for (int wi = w0; wi < w1; ++wi) {
    uint32_t m = __ldcg(bits + wi);
    while (m) {
      const int b = __ffs(m) - 1;
      m &= m - 1;
      if (pos < static_cast<uint32_t>(K)) out[pos] = wi * 32 + b;
      ++pos;
    }
  }
  if (tid == 0 && (total != static_cast<uint32_t>(K) || cand_n > kCandCap)) record_status(p.status, kStatusDeviceArg);
  for (int j = static_cast<int>(total) + tid; j < K; j += kThreads) out[j] = -1;
}

}  // namespace

size_t topk_bitmap_words(int kv_stride) { return (static_cast<size_t>(kv_stride) + 31) / 32; }

// CTAs per query: enough to fill the GPU once, at most kMaxCluster.
int topk_cluster_size(int rows) {
  int c = 1;
  while (c < kMaxCluster && static_cast<long long>(rows) * c * 2 <= 148) c *= 2;
  return c;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t stream) {
  if (a.rows == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(sga_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSmemBytes));
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
  const int C = topk_cluster_size(a.rows);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.rows * C));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sga_topk_kernel, p);
}

}  // namespace sga
