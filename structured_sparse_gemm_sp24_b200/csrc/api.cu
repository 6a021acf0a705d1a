// libsp24: size queries, status word, error strings, device checks.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "sp24_device.cuh"
#include "sp24_host.h"

namespace sp24 {

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];   // 0 unknown, 1 sm_100, 2 other
std::atomic<int> g_dev_sms[kMaxDevices];
std::mutex g_dev_mu;
}  // namespace

namespace {
thread_local char g_last_err[256] = "";
}  // namespace

// Status-word bit of sp24_permute_columns: a permutation entry outside
// [0, K) (the pattern and timeout bits sit with the status word itself).
constexpr uint32_t kErrIndexBit = 4u;
static_assert((kErrIndexBit & (kErrPatternBit | kErrTimeoutBit)) == 0, "status bits overlap");

sp24_status cuda_fail(const char* what, const char* err_name) {
  std::snprintf(g_last_err, sizeof(g_last_err), "%s: %s", what, err_name ? err_name : "?");
  return SP24_ERR_CUDA;
}

sp24_status check_device() {
  g_last_err[0] = '\0';
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kMaxDevices) return SP24_ERR_UNSUPPORTED;
  int ok = g_dev_ok[dev].load();
  if (ok == 0) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    ok = g_dev_ok[dev].load();
    if (ok == 0) {
      int major = 0, sms = 0;
      cudaError_t a = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
      if (a == cudaSuccess) a = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (a != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", a);
      g_dev_sms[dev].store(sms);   // before the flag: sm_count() may read it next
      ok = (major == 10) ? 1 : 2;
      g_dev_ok[dev].store(ok);
    }
  }
  return ok == 1 ? SP24_OK : SP24_ERR_UNSUPPORTED;
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDevices) return 148;
  const int sms = g_dev_sms[dev].load();
  return sms > 0 ? sms : 148;
}

// One thread waits, with a bounded wait of limit_ns, on an mbarrier that
// nothing arrives at: the wait gives up, records SP24_ERR_TIMEOUT in the
// status word and the kernel returns normally.
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  mbar_wait_limit(&bar, 0, limit_ns);
}

}  // namespace sp24

using namespace sp24;

extern "C" {

size_t sp24_mask_bytes(int64_t N, int64_t K) {
  if (N < 0 || K < 0 || (K % 8) != 0) return 0;
  return static_cast<size_t>(N) * static_cast<size_t>(K / 8);
}

size_t sp24_vals_bytes(int64_t N, int64_t K, int dtype) {
  if (N < 0 || K < 0 || (K % 8) != 0) return 0;
  const size_t el = dtype == SP24_BF16 ? 2 : (dtype == SP24_INT8 ? 1 : 0);
  return static_cast<size_t>(N) * static_cast<size_t>(K / 2) * el;
}

size_t sp24_meta_bytes(int64_t N, int64_t K) {
  if (N < 0 || K < 0 || (K % 8) != 0) return 0;
  const size_t nr = static_cast<size_t>((N + 127) / 128);
  const size_t kc = static_cast<size_t>((K + 127) / 128);
  return nr * kc * 2048u;
}

size_t sp24_prune_workspace_bytes(int64_t K, int mode) {
  if (K < 0) return 0;
  return mode == SP24_WANDA ? static_cast<size_t>(K) * sizeof(double) : 0;
}

sp24_status sp24_selftest_wait_timeout(int64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 1000000000) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  selftest_wait_kernel<<<1, 1, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_ns));
  return launch_status();
}

sp24_status sp24_device_status(void* stream) {
  g_last_err[0] = '\0';
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail("cudaStreamSynchronize", e);
  uint32_t word = 0;
  e = cudaMemcpyFromSymbol(&word, g_status, sizeof(word));
  if (e != cudaSuccess) return cuda_fail("cudaMemcpyFromSymbol", e);
  if (word != 0) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(g_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyToSymbol", e);
  }
  if (word & kErrTimeoutBit) return SP24_ERR_TIMEOUT;
  if (word & kErrPatternBit) return SP24_ERR_PATTERN;
  if (word & kErrIndexBit) return SP24_ERR_INDEX;
  return SP24_OK;
}

const char* sp24_strerror(int status) {
  switch (status) {
    case SP24_OK: return "ok";
    case SP24_ERR_ARG: return "invalid argument (null pointer, negative size or unknown enum)";
    case SP24_ERR_ALIGN: return "alignment rule broken (sizes or 16-byte pointer alignment)";
    case SP24_ERR_PATTERN: return "a group of 4 does not keep exactly two positions";
    case SP24_ERR_CUDA: return "CUDA runtime error";
    case SP24_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case SP24_ERR_UNSUPPORTED: return "unsupported device or argument combination";
    case SP24_ERR_INDEX: return "a permutation entry lies outside [0, K)";
    default: return "unknown status";
  }
}

int sp24_version(void) { return 300; }

const char* sp24_last_cuda_error(void) { return g_last_err; }

}  // extern "C"
