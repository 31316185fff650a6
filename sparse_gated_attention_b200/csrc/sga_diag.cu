// Diagnostic of the device-side failure path of the kernels: a bounded wait
// that runs out, the status word it writes, and the unwind after it.
//
// Every wait inside the path's kernels (mbar_wait in sga_ptx.cuh) has a cycle
// budget and watches an abort flag shared by its CTA.  When one runs out, the
// waiting thread records SGA_ERR_TIMEOUT in the workspace status word and
// raises the flag, so every other wait of the CTA returns at once; the CTA then
// frees its tensor memory and exits.  This kernel runs exactly that sequence on
// a barrier that nothing ever completes, with no copy in flight: warp 0 waits
// with the caller's short budget, warp 1 with the path's own budget (about a
// second) and is released only by the abort flag.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sga.h"
#include "sga_host.h"
#include "sga_ptx.cuh"

namespace sga {
namespace {

constexpr uint32_t kDiagTmemCols = 32;  // the smallest tensor-memory allocation

__global__ void __launch_bounds__(64, 1) bounded_wait_selftest_kernel(int* status, long long budget) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // one arrival expected; none ever comes
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_slot), kDiagTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  volatile int* flag = &abort_flag;
  if (lane == 0) {
    const bool done = warp == 0 ? mbar_wait(smem_u32(&bar), 0, flag, budget) : mbar_wait(smem_u32(&bar), 0, flag);
    if (!done) {
      record_status(status, kStatusTimeout);
      *flag = 1;
      atomicAdd(status + 1, 1);  // waits that gave up
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_slot, kDiagTmemCols);
  }
}

}  // namespace
}  // namespace sga

extern "C" {

sga_status_t sga_selftest_bounded_wait(int64_t budget_cycles, void* ws, size_t ws_bytes, sga_stream_t stream) {
  if (budget_cycles < 1 || budget_cycles >= (int64_t{1} << 31)) return SGA_ERR_INVALID_ARG;
  if (!sga::host::aligned(ws, sga::host::kWsAlign) || ws_bytes < sga::host::kStatusBytes) return SGA_ERR_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return SGA_ERR_UNSUPPORTED;
  }
  sga::bounded_wait_selftest_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(
      sga::host::at<int>(ws, 0), static_cast<long long>(budget_cycles));
  if (cudaGetLastError() != cudaSuccess) return SGA_ERR_CUDA;
  return SGA_OK;
}

}  // extern "C"
