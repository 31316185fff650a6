// Host-side helpers shared by the C-ABI entry points: workspace alignment,
// the status block at the start of every workspace, pointer checks.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stddef.h>
#include <stdint.h>

namespace sga {
namespace host {

constexpr size_t kWsAlign = 256;      // every workspace region starts on this boundary
constexpr size_t kStatusBytes = 256;  // the status block at the start of a workspace

inline size_t align_up(size_t x) { return (x + kWsAlign - 1) / kWsAlign * kWsAlign; }

// Non-null and a multiple of `a` bytes.
inline bool aligned(const void* p, size_t a) { return p && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// The region of the workspace `off` bytes from its start.
template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// One NVTX range (named after the stage it brackets) for the lifetime of the
// object: the host-side launch of that stage shows as a range in profilers.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Launches `kernel` with programmatic dependent launch: its grid may be
// scheduled once every CTA of the previous kernel on the stream has called
// griddepcontrol.launch_dependents (or exited), so its set-up overlaps that
// kernel's tail; its griddepcontrol.wait orders the reads that depend on it.
template <class... Params, class... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace host
}  // namespace sga
