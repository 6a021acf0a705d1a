// libsp24: 3x3 convolution input as the sparse GEMM's token operand
// ([Orin ch.7] 2.2 A.3: large 3x3 convolutions at large batch or high
// resolution are good 2:4 candidates; 2.1: groups of 4 along the input
// channels).  Stride 1, zero padding 1, NHWC activations.
//
// A[(b*H + h)*W + w][(kh*3 + kw)*C + c] = X[b][h+kh-1][w+kw-1][c], 0 outside
// the image, so that Y = A * W'^T with W[Cout][3][3][C] pruned and compressed
// as [Cout][9*C] is the convolution (groups of 4 stay inside one tap when
// C % 4 == 0).  This gather writes A to memory (9x the activation bytes); the
// GEMM then reads it like any token operand.
#include <algorithm>

#include "sp24_device.cuh"
#include "sp24_host.h"

namespace sp24 {
namespace conv {

// One 16-byte vector of A per thread and iteration; cv = vectors per pixel
// and tap (C * element bytes / 16).
__global__ void __launch_bounds__(256) im2col3x3_kernel(const uint4* __restrict__ x, int64_t hh,
                                                        int64_t ww, int64_t cv, int64_t total,
                                                        uint4* __restrict__ a) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const int64_t rowv = 9 * cv;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * 256) {
    const int64_t m = e / rowv;
    const int64_t j = e - m * rowv;
    const int tap = static_cast<int>(j / cv);
    const int64_t v = j - tap * cv;
    const int64_t w = m % ww;
    const int64_t t = m / ww;
    const int64_t h = t % hh;
    const int64_t b = t / hh;
    const int64_t ih = h + tap / 3 - 1;
    const int64_t iw = w + tap % 3 - 1;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (ih >= 0 && ih < hh && iw >= 0 && iw < ww) val = __ldg(x + ((b * hh + ih) * ww + iw) * cv + v);
    __stcs(a + e, val);
  }
}

}  // namespace conv
}  // namespace sp24

using namespace sp24;

extern "C" {

sp24_status sp24_im2col3x3(const void* X, int64_t B, int64_t H, int64_t W, int64_t C,
                           int elem_bytes, void* A, void* stream) {
  if (B < 0 || H < 0 || W < 0 || C < 0) return SP24_ERR_ARG;
  if (elem_bytes != 1 && elem_bytes != 2) return SP24_ERR_ARG;
  if (B == 0 || H == 0 || W == 0 || C == 0) return SP24_OK;
  if (!X || !A) return SP24_ERR_ARG;
  if ((C * elem_bytes) % 16 != 0 || !aligned16(X) || !aligned16(A)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  const int64_t cv = C * elem_bytes / 16;
  const int64_t total = B * H * W * 9 * cv;
  const int64_t blocks = std::min<int64_t>((total + 255) / 256, 16 * static_cast<int64_t>(sm_count()));
  return launch_kernel(conv::im2col3x3_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                       as_stream(stream), 1, static_cast<const uint4*>(X), H, W, cv, total,
                       static_cast<uint4*>(A));
}

}  // extern "C"
