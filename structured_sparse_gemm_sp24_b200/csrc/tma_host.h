// Host helpers for TMA tensor maps (driver entry point looked up through the
// runtime, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "sp24_host.h"

namespace sp24 {

inline PFN_cuTensorMapEncodeTiled_v12000& tma_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

inline bool get_encoder() { return tma_encoder() != nullptr; }

// 2D row-major [rows][cols] map with a {box_cols, box_rows} box, zero fill
// outside the tensor.
inline sp24_status make_map(CUtensorMap* map, const void* base, CUtensorMapDataType dt,
                            int elsize, uint64_t cols, uint64_t rows, uint32_t box_cols,
                            uint32_t box_rows,
                            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!get_encoder()) return cuda_fail("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elsize)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = tma_encoder()(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r == CUDA_SUCCESS) return SP24_OK;
  char buf[96];
  std::snprintf(buf, sizeof(buf), "CUresult %d (box %ux%u, dims %llux%llu)", static_cast<int>(r),
                box_cols, box_rows, static_cast<unsigned long long>(cols),
                static_cast<unsigned long long>(rows));
  return cuda_fail("cuTensorMapEncodeTiled", buf);
}

// 4D map over an NHWC activation tensor [b][h][w][c] (dims innermost first:
// c, w, h, b) with a {box_c, box_w, box_h, 1} box, 128-byte swizzle and zero
// fill outside the tensor (the implicit convolution's padding).
inline sp24_status make_map_nhwc(CUtensorMap* map, const void* base, CUtensorMapDataType dt,
                                 int elsize, uint64_t c, uint64_t w, uint64_t h, uint64_t b,
                                 uint32_t box_c, uint32_t box_w, uint32_t box_h) {
  if (!get_encoder()) return cuda_fail("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled");
  const uint64_t es = static_cast<uint64_t>(elsize);
  cuuint64_t dims[4] = {c, w, h, b};
  cuuint64_t strides[3] = {c * es, w * c * es, h * w * c * es};
  cuuint32_t box[4] = {box_c, box_w, box_h, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = tma_encoder()(map, dt, 4, const_cast<void*>(base), dims, strides, box, estr,
                                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r == CUDA_SUCCESS) return SP24_OK;
  char buf[112];
  std::snprintf(buf, sizeof(buf), "CUresult %d (nhwc box %ux%ux%u, dims %llux%llux%llux%llu)",
                static_cast<int>(r), box_c, box_w, box_h, static_cast<unsigned long long>(c),
                static_cast<unsigned long long>(w), static_cast<unsigned long long>(h),
                static_cast<unsigned long long>(b));
  return cuda_fail("cuTensorMapEncodeTiled", buf);
}

// 1D map over `len` elements with a `box`-element box, zero fill past the end.
inline sp24_status make_map_1d(CUtensorMap* map, const void* base, CUtensorMapDataType dt,
                               uint64_t len, uint32_t box) {
  if (!get_encoder()) return cuda_fail("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled");
  cuuint64_t dims[1] = {len};
  cuuint64_t strides[1] = {0};
  cuuint32_t boxd[1] = {box};
  cuuint32_t estr[1] = {1};
  const CUresult r = tma_encoder()(map, dt, 1, const_cast<void*>(base), dims, strides, boxd,
                                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                   CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r == CUDA_SUCCESS) return SP24_OK;
  char buf[80];
  std::snprintf(buf, sizeof(buf), "CUresult %d (1d box %u, len %llu)", static_cast<int>(r), box,
                static_cast<unsigned long long>(len));
  return cuda_fail("cuTensorMapEncodeTiled", buf);
}

}  // namespace sp24
