// Step 2: top-K selection (archdb "A.X K2", token-selection field: top-2048
// tokens per query; arXiv abstract "A.X K2 Technical Report": each query reads
// only 2,048 positions).  Larger score first; equal scores go to the lower
// position; output ascending, -1 padded.
//
// Each candidate s gets a unique 64-bit key
//     (order-preserving bits of score[s]) << 32  |  (0xFFFFFFFF - s)
// so "larger key" is exactly the selection order and the K-th largest key is a
// single threshold.  One 1024-thread CTA per query:
//   1. MSD radix select over the keys, 11 bits per level: a shared-memory
//      histogram (warp-aggregated with __match_any_sync) of the next digit
//      among keys that share the prefix found so far, a block scan from the
//      top bin, then narrow.  Stop as soon as the bucket holding the threshold
//      fits the shared-memory candidate list (usually after 1-2 passes).
//   2. One pass that writes a selection bitmap (a warp ballot per 32
//      positions) for every key above the bucket and appends the bucket's keys
//      to the candidate list.
//   3. Finish the radix select on the candidate list in shared memory and set
//      the bits of the chosen candidates.
//   4. Emit: per-thread popcounts over the bitmap words, a block scan, and each
//      thread writes its set bits in position order.
#include "sga_internal.cuh"
#include "sga_ptx.cuh"

namespace sga {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kCandCap = 8192;
constexpr size_t kSmemBytes = kBins * 4 + kCandCap * 8 + 256;

struct TopkParams {
  const float* scores;
  const int32_t* q_pos;
  int32_t* idx;
  uint32_t* bitmap;
  int* status;
  int kv_stride, top_k;
  long long words_per_row;
};

__device__ __forceinline__ uint32_t order_bits(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0.0 ranks as +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

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

// Finds the bin holding the `need`-th largest key: counts in bins above it are
// < need <= counts in bins at or above it.  Bins are scanned from the top.
__device__ __forceinline__ Narrow find_bin(const uint32_t* hist, uint32_t need, uint32_t* warp_buf, Narrow* out) {
  const int i = threadIdx.x;
  const int hi_bin = kBins - 1 - 2 * i, lo_bin = kBins - 2 - 2 * i;
  const uint32_t h_hi = hist[hi_bin], h_lo = hist[lo_bin];
  uint32_t total;
  const uint32_t incl = block_inclusive_scan(h_hi + h_lo, warp_buf, total);
  const uint32_t excl = incl - h_hi - h_lo;
  if (excl < need && need <= incl) {
    if (excl + h_hi >= need) {
      out->digit = hi_bin;
      out->above = excl;
      out->count = h_hi;
    } else {
      out->digit = lo_bin;
      out->above = excl + h_hi;
      out->count = h_lo;
    }
  }
  __syncthreads();
  return *out;
}

__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t key = active ? bin : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xFFFFFFFFu, key);
  const int lane = threadIdx.x & 31;
  if (active && lane == __ffs(peers) - 1) atomicAdd(hist + bin, static_cast<uint32_t>(__popc(peers)));
}

__global__ void __launch_bounds__(kThreads, 1) sga_topk_kernel(TopkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem_raw + kBins * 4);
  __shared__ uint32_t warp_buf[kWarps];
  __shared__ Narrow narrow;
  __shared__ uint32_t cand_n;

  const int row = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.top_k;
  int32_t* out = p.idx + static_cast<size_t>(row) * K;
  const int t = __ldg(p.q_pos + row);
  if (t < 0 || t >= p.kv_stride) {
    if (tid == 0) record_status(p.status, kStatusDeviceArg);
    for (int j = tid; j < K; j += kThreads) out[j] = -1;
    return;
  }
  const int n = t + 1;
  if (n <= K) {
    for (int j = tid; j < K; j += kThreads) out[j] = j < n ? j : -1;
    return;
  }
  const float* sc = p.scores + static_cast<size_t>(row) * p.kv_stride;
  uint32_t* bits = p.bitmap + static_cast<size_t>(row) * p.words_per_row;

  // ---- 1. radix levels over the full row until the threshold bucket is small
  uint64_t prefix = 0, mask = 0;
  uint32_t need = static_cast<uint32_t>(K);
  int shift = 64;
  uint32_t bucket = 0;
  while (true) {
    const int width = shift >= 11 ? 11 : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kThreads) {
      const int s = base + tid;
      bool act = false;
      uint32_t bin = 0;
      if (s < n) {
        const uint64_t c = sel_key(__ldg(sc + s), s);
        act = (c & mask) == prefix;
        bin = static_cast<uint32_t>(c >> shift) & dmask;
      }
      hist_add(hist, bin, act);
    }
    __syncthreads();
    const Narrow nr = find_bin(hist, need, warp_buf, &narrow);
    prefix |= static_cast<uint64_t>(nr.digit) << shift;
    mask |= static_cast<uint64_t>(dmask) << shift;
    need -= nr.above;
    bucket = nr.count;
    if (bucket <= kCandCap || shift == 0) break;
  }

  // ---- 2. bitmap of keys above the bucket; bucket keys -> candidate list
  if (tid == 0) cand_n = 0;
  __syncthreads();
  for (int base = 0; base < n; base += kThreads) {
    const int s = base + tid;
    bool above = false, in_bucket = false;
    uint64_t c = 0;
    if (s < n) {
      c = sel_key(__ldg(sc + s), s);
      above = (c & mask) > prefix;
      in_bucket = (c & mask) == prefix;
    }
    const uint32_t word = __ballot_sync(0xFFFFFFFFu, above);
    const int first = base + warp * 32;
    if (lane == 0 && first < n) bits[first >> 5] = word;
    const uint32_t cm = __ballot_sync(0xFFFFFFFFu, in_bucket);
    if (cm) {
      uint32_t off = 0;
      if (lane == 0) off = atomicAdd(&cand_n, static_cast<uint32_t>(__popc(cm)));
      off = __shfl_sync(0xFFFFFFFFu, off, 0);
      if (in_bucket) {
        const uint32_t r = off + __popc(cm & ((1u << lane) - 1u));
        if (r < kCandCap) cand[r] = c;
      }
    }
  }
  __syncthreads();
  const uint32_t nc = cand_n < kCandCap ? cand_n : kCandCap;

  // ---- 3. finish the select inside the candidate list
  while (need < bucket && shift > 0) {
    const int width = shift >= 11 ? 11 : shift;
    shift -= width;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += kThreads) hist[b] = 0;
    __syncthreads();
    for (uint32_t base = 0; base < nc; base += kThreads) {
      const uint32_t i = base + tid;
      bool act = false;
      uint32_t bin = 0;
      if (i < nc) {
        const uint64_t c = cand[i];
        act = (c & mask) == prefix;
        bin = static_cast<uint32_t>(c >> shift) & dmask;
      }
      hist_add(hist, bin, act);
    }
    __syncthreads();
    const Narrow nr = find_bin(hist, need, warp_buf, &narrow);
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

  // ---- 4. emit set bits in position order
  const int words = (n + 31) >> 5;
  const int per = (words + kThreads - 1) / kThreads;
  const int w0 = min(tid * per, words), w1 = min(w0 + per, words);
  uint32_t cnt = 0;
  for (int wi = w0; wi < w1; ++wi) cnt += __popc(bits[wi]);
  uint32_t total;
  uint32_t pos = block_inclusive_scan(cnt, warp_buf, total) - cnt;
  for (int wi = w0; wi < w1; ++wi) {
    uint32_t m = bits[wi];
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
  p.status = a.status;
  p.kv_stride = a.kv_stride;
  p.top_k = a.top_k;
  p.words_per_row = static_cast<long long>(topk_bitmap_words(a.kv_stride));
  sga_topk_kernel<<<a.rows, kThreads, kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace sga
