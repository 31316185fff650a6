// C ABI of libsga: argument validation, workspace layout, tensor-map encoding
// and kernel launches.  See include/sga.h for the contract of each call.
#include <cudaTypedefs.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/sga.h"
#include "sga_host.h"
#include "sga_internal.cuh"

namespace sga {
namespace {

using host::align_up;
using host::aligned;
using host::at;
using host::kStatusBytes;
constexpr size_t kAlign = host::kWsAlign;

struct Layout {
  size_t bitmap = 0, scores = 0, idx = 0, hist = 0, cand = 0, cand_n = 0, total = 0;
};

bool dims_ok(const sga_dims_t* d) {
  if (!d) return false;
  if (d->batch < 1 || d->n_q < 1 || d->kv_stride < 1 || d->kv_stride > SGA_MAX_KV_STRIDE) return false;
  if (d->top_k < 64 || d->top_k > SGA_MAX_TOP_K || d->top_k % 64 != 0) return false;
  const long long rows = static_cast<long long>(d->batch) * d->n_q;
  // row indices of the flattened [rows*64] query matrices and [B*L] caches are int32
  if (rows * 64 > INT32_MAX || static_cast<long long>(d->batch) * d->kv_stride > INT32_MAX) return false;
  return true;
}

Layout make_layout(const sga_dims_t& d, sga_op_t op) {
  Layout l;
  const size_t rows = static_cast<size_t>(d.batch) * d.n_q;
  size_t off = kStatusBytes;
  if (op == SGA_OP_FORWARD_FUSED && fused_topk_ok(d.n_q, d.kv_stride)) {
    // no scores and no bitmaps: up to L candidates of 8 bytes per row, and the
    // rows' candidate counters
    l.idx = off;
    off += align_up(rows * static_cast<size_t>(d.top_k) * 4);
    l.hist = off;
    off += align_up(rows * 4096 * 4);
    l.cand = off;
    off += align_up(rows * static_cast<size_t>(d.kv_stride) * 8);
    l.cand_n = off;
    off += align_up(rows * kCandNStride * 4);
    l.total = off;
    return l;
  }
  if (op == SGA_OP_FORWARD_FUSED) op = SGA_OP_FORWARD;  // rows the fused selection does not take
  if (op == SGA_OP_TOPK_SELECT || op == SGA_OP_FORWARD) {
    l.bitmap = off;
    off += align_up(rows * 2 * topk_bitmap_words(d.kv_stride) * 4);  // selection + tie bitmaps
  }
  // The attention needs no workspace beyond the status word: the splits of a
  // query merge their partial results on chip.
  if (op == SGA_OP_FORWARD) {
    l.scores = off;
    off += align_up(rows * static_cast<size_t>(d.kv_stride) * 4);
    l.idx = off;
    off += align_up(rows * static_cast<size_t>(d.top_k) * 4);
    l.hist = off;
    off += align_up(rows * 4096 * 4);
  }
  l.total = off;
  return l;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

// Checks that the current device is an sm_100 part and returns its SM count.
sga_status_t device_info(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  if (major != 10) return SGA_ERR_UNSUPPORTED;
  *num_sms = sms;
  return SGA_OK;
}

sga_status_t check_ws(void* ws, size_t ws_bytes, const sga_dims_t& d, sga_op_t op, Layout* l) {
  *l = make_layout(d, op);
  if (!ws || !aligned(ws, kAlign)) return SGA_ERR_WORKSPACE;
  if (ws_bytes < l->total) return SGA_ERR_WORKSPACE;
  return SGA_OK;
}

// A failed launch or runtime call also leaves the error as the thread's last
// CUDA error; it is cleared here so that it does not surface in the caller's
// next, unrelated error check.
sga_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return SGA_OK;
  cudaGetLastError();
  return SGA_ERR_CUDA;
}

}  // namespace

// 2-D tiled tensor map with the 128-byte swizzle over a row-major [outer][inner] array.
cudaError_t make_tmap_2d(CUtensorMap* map, bool bytes, const void* base, uint64_t inner, uint64_t outer,
                         uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  std::call_once(g_encode_once, []() {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cudaGetLastError();
  });
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  return make_tmap_2d(map, false, base, inner, outer, row_bytes, box_inner, box_outer);
}

}  // namespace sga

using namespace sga;

namespace {

// The indexer with bf16 or E4M3 (fp8) queries and keys; the rest of the path is shared.
sga_status_t index_scores_impl(const sga_dims_t* dims, const void* q_idx, const sga_bf16_t* w, const void* k_idx,
                               const int32_t* q_pos, float* scores, void* ws, size_t ws_bytes, sga_stream_t stream,
                               bool fp8) {
  if (!dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(w, 16) || !aligned(k_idx, 16) || !aligned(q_pos, 4) || !aligned(scores, 16))
    return SGA_ERR_INVALID_ARG;
  Layout l;
  sga_status_t st = check_ws(ws, ws_bytes, *dims, SGA_OP_INDEX_SCORES, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_info(&sms)) != SGA_OK) return st;
  host::NvtxRange range("sga.index_scores");
  IndexArgs a{q_idx, w, k_idx, q_pos, scores, nullptr, at<int>(ws, 0), dims->batch, dims->n_q, dims->kv_stride, fp8};
  return from_cuda(launch_index_scores(a, sms, static_cast<cudaStream_t>(stream)));
}

sga_status_t forward_impl(const sga_dims_t* dims, const void* q_idx, const sga_bf16_t* w, const void* k_idx,
                          const sga_bf16_t* q, const sga_bf16_t* kv, const sga_bf16_t* gate, const int32_t* q_pos,
                          int32_t* idx_out, float* out, void* ws, size_t ws_bytes, sga_stream_t stream, bool fp8,
                          bool fused, uint16_t* out_bf16 = nullptr) {
  if (!dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(q_idx, 16) || !aligned(w, 16) || !aligned(k_idx, 16) || !aligned(q, 16) || !aligned(kv, 16) ||
      !aligned(q_pos, 4) || !aligned(out, 16) || (gate && !aligned(gate, 2)) || (idx_out && !aligned(idx_out, 16)) ||
      (out_bf16 && !aligned(out_bf16, 8)))
    return SGA_ERR_INVALID_ARG;
  Layout l;
  sga_status_t st = check_ws(ws, ws_bytes, *dims, fused ? SGA_OP_FORWARD_FUSED : SGA_OP_FORWARD, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_info(&sms)) != SGA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The fused selection: the indexer writes no scores; it keeps a running
  // per-row threshold from the histogram counted so far and appends only the
  // keys that can still be selected, and the selection reads those (clearing
  // their counters for the next call).
  const bool cand_mode = fused && fused_topk_ok(dims->n_q, dims->kv_stride);
  int* status = at<int>(ws, 0);
  float* scores = at<float>(ws, l.scores);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, l.idx);
  const int rows = dims->batch * dims->n_q;
  // The indexer counts the first radix level of the selection as it writes the
  // scores; the selection clears each histogram row after reading it, so a
  // zero-filled workspace stays ready for the next call.
  uint32_t* hist = index_uses_prefill(dims->n_q) ? nullptr : at<uint32_t>(ws, l.hist);
  cudaError_t e;
  {
    host::NvtxRange range("sga.index_scores");
    IndexArgs ia{q_idx, w, k_idx, q_pos, scores, hist, status, dims->batch, dims->n_q, dims->kv_stride, fp8};
    if (cand_mode) {
      ia.scores = nullptr;
      ia.cand = at<uint64_t>(ws, l.cand);
      ia.cand_n = at<uint32_t>(ws, l.cand_n);
      ia.top_k = dims->top_k;
    }
    e = launch_index_scores(ia, sms, s);
  }
  if (e != cudaSuccess) return from_cuda(e);
  {
    host::NvtxRange range("sga.topk_select");
    if (cand_mode) {
      TopkCandArgs ca{at<uint64_t>(ws, l.cand), at<uint32_t>(ws, l.cand_n), hist, q_pos, idx, status, rows,
                      dims->kv_stride, dims->top_k};
      e = launch_topk_candidates(ca, s);
    } else {
      TopkArgs ta{scores, q_pos, idx, at<uint32_t>(ws, l.bitmap), hist, status, rows, dims->kv_stride, dims->top_k};
      e = launch_topk(ta, s);
    }
  }
  if (e != cudaSuccess) return from_cuda(e);
  host::NvtxRange range("sga.sparse_mla_attend");
  AttendArgs aa{q, kv, idx, gate, out, status, dims->batch, dims->n_q, dims->kv_stride, dims->top_k};
  aa.out_bf16 = out_bf16;
  return from_cuda(launch_attend(aa, s));
}

}  // namespace

namespace sga {
sga_status_t forward_bf16_copy(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                               const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                               const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out,
                               uint16_t* out_bf16, void* ws, size_t ws_bytes, sga_stream_t stream) {
  return forward_impl(dims, q_idx, w, k_idx, q, kv, gate, q_pos, idx_out, out, ws, ws_bytes, stream, false, false,
                      out_bf16);
}
}  // namespace sga


extern "C" {

int32_t sga_abi_version(void) { return 1; }

const char* sga_status_string(sga_status_t s) {
  switch (s) {
    case SGA_OK: return "SGA_OK";
    case SGA_ERR_INVALID_ARG: return "SGA_ERR_INVALID_ARG";
    case SGA_ERR_UNSUPPORTED: return "SGA_ERR_UNSUPPORTED";
    case SGA_ERR_WORKSPACE: return "SGA_ERR_WORKSPACE";
    case SGA_ERR_CUDA: return "SGA_ERR_CUDA";
    case SGA_ERR_TIMEOUT: return "SGA_ERR_TIMEOUT";
    case SGA_ERR_DEVICE_ARG: return "SGA_ERR_DEVICE_ARG";
    case SGA_ERR_INTERNAL: return "SGA_ERR_INTERNAL";
  }
  return "SGA_ERR_UNKNOWN";
}

sga_status_t sga_workspace_size(const sga_dims_t* dims, sga_op_t op, size_t* bytes) {
  if (!dims_ok(dims) || !bytes || op < SGA_OP_INDEX_SCORES || op > SGA_OP_FORWARD_FUSED) return SGA_ERR_INVALID_ARG;
  *bytes = make_layout(*dims, op).total;
  return SGA_OK;
}


sga_status_t sga_index_scores(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                              const sga_bf16_t* k_idx, const int32_t* q_pos, float* scores, void* ws,
                              size_t ws_bytes, sga_stream_t stream) {
  return index_scores_impl(dims, q_idx, w, k_idx, q_pos, scores, ws, ws_bytes, stream, false);
}

sga_status_t sga_index_scores_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx, const sga_bf16_t* w,
                                  const sga_fp8_e4m3_t* k_idx, const int32_t* q_pos, float* scores, void* ws,
                                  size_t ws_bytes, sga_stream_t stream) {
  return index_scores_impl(dims, q_idx, w, k_idx, q_pos, scores, ws, ws_bytes, stream, true);
}

sga_status_t sga_topk_select(const sga_dims_t* dims, const float* scores, const int32_t* q_pos, int32_t* idx,
                             void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (!dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(q_pos, 4) || !aligned(idx, 16)) return SGA_ERR_INVALID_ARG;
  Layout l;
  sga_status_t st = check_ws(ws, ws_bytes, *dims, SGA_OP_TOPK_SELECT, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_info(&sms)) != SGA_OK) return st;
  host::NvtxRange range("sga.topk_select");
  TopkArgs a{scores,          q_pos, idx, at<uint32_t>(ws, l.bitmap), nullptr, at<int>(ws, 0),
             dims->batch * dims->n_q, dims->kv_stride, dims->top_k};
  return from_cuda(launch_topk(a, static_cast<cudaStream_t>(stream)));
}

sga_status_t sga_sparse_mla_attend(const sga_dims_t* dims, const sga_bf16_t* q, const sga_bf16_t* kv,
                                   const int32_t* idx, const sga_bf16_t* gate, float* out, void* ws,
                                   size_t ws_bytes, sga_stream_t stream) {
  if (!dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv, 16) || !aligned(idx, 16) || !aligned(out, 16) ||
      (gate && !aligned(gate, 2)))
    return SGA_ERR_INVALID_ARG;
  Layout l;
  sga_status_t st = check_ws(ws, ws_bytes, *dims, SGA_OP_SPARSE_MLA_ATTEND, &l);
  if (st != SGA_OK) return st;
  int sms = 0;
  if ((st = device_info(&sms)) != SGA_OK) return st;
  host::NvtxRange range("sga.sparse_mla_attend");
  AttendArgs a{q, kv, idx, gate, out, at<int>(ws, 0), dims->batch, dims->n_q, dims->kv_stride, dims->top_k};
  return from_cuda(launch_attend(a, static_cast<cudaStream_t>(stream)));
}


sga_status_t sga_forward(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                         const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                         const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out, void* ws,
                         size_t ws_bytes, sga_stream_t stream) {
  return forward_impl(dims, q_idx, w, k_idx, q, kv, gate, q_pos, idx_out, out, ws, ws_bytes, stream, false, false);
}

sga_status_t sga_forward_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx, const sga_bf16_t* w,
                             const sga_fp8_e4m3_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                             const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out, void* ws,
                             size_t ws_bytes, sga_stream_t stream) {
  return forward_impl(dims, q_idx, w, k_idx, q, kv, gate, q_pos, idx_out, out, ws, ws_bytes, stream, true, false);
}

sga_status_t sga_forward_fused(const sga_dims_t* dims, const sga_bf16_t* q_idx, const sga_bf16_t* w,
                               const sga_bf16_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                               const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out,
                               void* ws, size_t ws_bytes, sga_stream_t stream) {
  return forward_impl(dims, q_idx, w, k_idx, q, kv, gate, q_pos, idx_out, out, ws, ws_bytes, stream, false, true);
}

sga_status_t sga_forward_fused_fp8(const sga_dims_t* dims, const sga_fp8_e4m3_t* q_idx, const sga_bf16_t* w,
                                   const sga_fp8_e4m3_t* k_idx, const sga_bf16_t* q, const sga_bf16_t* kv,
                                   const sga_bf16_t* gate, const int32_t* q_pos, int32_t* idx_out, float* out,
                                   void* ws, size_t ws_bytes, sga_stream_t stream) {
  return forward_impl(dims, q_idx, w, k_idx, q, kv, gate, q_pos, idx_out, out, ws, ws_bytes, stream, true, true);
}

sga_status_t sga_get_device_status(const void* ws, sga_stream_t stream, int32_t* device_status) {
  if (!ws || !device_status) return SGA_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return SGA_ERR_CUDA;
  }
  *device_status = v;
  return SGA_OK;
}

sga_status_t sga_clear_device_status(void* ws, sga_stream_t stream) {
  if (!ws) return SGA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, kStatusBytes, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---- top-k without a caller workspace -------------------------------------------------
// Scratch of sga_topk_select_noalloc: a status word then the selection bitmaps.  It
// lives in the library for callers that cannot allocate device memory.  In host
// code the symbol is only a host-side stand-in, so the device address is looked
// up per device (with that device current) and passed to the kernel.  A lookup
// that fails is not remembered: the next call on that device tries again.
namespace {
constexpr int kNoallocMaxDevices = 64;
static __device__ __align__(256) unsigned char g_noalloc_scratch[SGA_NOALLOC_SCRATCH_BYTES];
void* g_noalloc_ptr[kNoallocMaxDevices] = {};
std::mutex g_noalloc_mu;

// The scratch array's device address on device `dev` (the current device), or null.
void* noalloc_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) == cudaSuccess) {
      g_noalloc_ptr[dev] = ptr;
    } else {
      cudaGetLastError();
    }
  }
  return g_noalloc_ptr[dev];
}
}  // namespace

extern "C" {

sga_status_t sga_topk_select_noalloc(const sga_dims_t* dims, const float* scores, const int32_t* q_pos,
                                     int32_t* idx, sga_stream_t stream) {
  if (!dims_ok(dims)) return SGA_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(q_pos, 4) || !aligned(idx, 16)) return SGA_ERR_INVALID_ARG;
  const size_t rows = static_cast<size_t>(dims->batch) * dims->n_q;
  const size_t bitmap_bytes = rows * 2 * topk_bitmap_words(dims->kv_stride) * 4;
  if (kStatusBytes + bitmap_bytes > SGA_NOALLOC_SCRATCH_BYTES) return SGA_ERR_WORKSPACE;
  int sms = 0;
  sga_status_t st = device_info(&sms);
  if (st != SGA_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  void* scratch = noalloc_scratch(dev);
  if (!scratch) return SGA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(scratch, 0, kStatusBytes, s);  // status word
  if (e != cudaSuccess) return from_cuda(e);
  TopkArgs a{scores,   q_pos, idx, at<uint32_t>(scratch, kStatusBytes), nullptr, at<int>(scratch, 0),
             static_cast<int>(rows), dims->kv_stride, dims->top_k};
  return from_cuda(launch_topk(a, s));
}

}  // extern "C"
