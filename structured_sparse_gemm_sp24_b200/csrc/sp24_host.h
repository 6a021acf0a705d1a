// Host-side helpers shared by the libsp24 translation units: argument
// checks, CUDA error mapping and the sm_100 device check.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/sp24.h"

namespace sp24 {

inline bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// SP24_OK when the current device is an sm_100 part (cached per device).
sp24_status check_device();

// Records a failed CUDA call for sp24_last_cuda_error() (thread-local) and
// returns SP24_ERR_CUDA.
sp24_status cuda_fail(const char* what, const char* err_name);
inline sp24_status cuda_fail(const char* what, cudaError_t e) {
  return cuda_fail(what, cudaGetErrorName(e));
}

// Maps the launch status of the last kernel to a library status.
inline sp24_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SP24_OK : cuda_fail("kernel launch", e);
}

// Number of SMs of the current device (cached).
int sm_count();

// Raises a kernel's dynamic shared-memory limit to `bytes` once per device.
// `done` holds one bit per device (0..63; check_device rejects others); two
// threads making the first call at once may both set it, which is harmless.
inline sp24_status set_smem_once(const void* kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return SP24_OK;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
  done.fetch_or(bit, std::memory_order_release);
  return SP24_OK;
}

// Launches every kernel of the library: programmatic stream serialization
// (the kernel may be scheduled while the previous kernel of the stream is
// finishing; each kernel of this library executes griddepcontrol.wait before
// it touches global memory, so it still sees all of that kernel's results)
// and, for cluster > 1, clusters of `cluster` CTAs along x.
template <class... KArgs, class... Args>
sp24_status launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return cuda_fail("cudaLaunchKernelEx", e);
  return launch_status();
}

}  // namespace sp24

#define SP24_TRY(expr)                    \
  do {                                    \
    sp24_status _st = (expr);             \
    if (_st != SP24_OK) return _st;       \
  } while (0)
