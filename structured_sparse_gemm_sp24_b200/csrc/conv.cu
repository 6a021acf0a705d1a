// libsp24: 3x3 convolution input as the sparse GEMM's token operand
// ([Orin ch.7] 2.2 A.3: large 3x3 convolutions at large batch or high
// resolution are good 2:4 candidates; 2.1: groups of 4 along the input
// channels).  Stride 1, zero padding 1, NHWC activations.
//
// A[(b*H + h)*W + w][(kh*3 + kw)*C + c] = X[b][h+kh-1][w+kw-1][c], 0 outside
// the image, so that Y = A * W'^T with W[Cout][3][3][C] pruned and compressed
// as [Cout][9*C] is the convolution (groups of 4 stay inside one tap when
// C % 4 == 0).  Two ways to run it:
//  * implicit GEMM (sp24_conv3x3): the CTA-pair sparse GEMM reads its token
//    tiles straight from X through a 4D tensor map (whole image rows per
//    tile, the tap's shift in the coordinates, the padding from the zero
//    fill), so A never exists in memory;
//  * explicit gather (sp24_im2col3x3) writes A to memory (9x the activation
//    bytes) for sp24_gemm, for shapes the implicit tiles do not cover.
#include <algorithm>

#include "sp24_device.cuh"
#include "sp24_host.h"
#include "tma_host.h"

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

// ------------------------------------------------- implicit GEMM launch
// Tile of the implicit convolution: whole image rows per CTA, in boxes of
// `rows` image rows such that rows * W is a multiple of 8 (1024-byte aligned
// boxes in the swizzled tile) and divides the CTA's tokens, and rows divides
// H (no box crosses an image); the tallest such box is used (fewest loads on
// the producer's path).  Up to 128 output channels: the single-SM
// kernel (128 weight rows, 128 or 112 tokens per tile); more: CTA pairs (256
// weight rows, 256 or 224 tokens per pair).  Among the tiles that fit, the
// one with the fewest k-block waves is taken (ties: the wider tile).
struct ConvTile {
  bool pair;
  int bn;      // tokens per tile
  int rows;
  int boxes;   // boxes per K-half of one CTA's tokens
};

bool conv_tile(int64_t m, int64_t n, int64_t h, int64_t w, ConvTile* t) {
  if (w < 1 || w > 256) return false;
  int units = sm_count();
  const bool pair = n > 128;
  if (pair && pair_capacity(&units) != SP24_OK) return false;
  const int64_t row_tiles = pair ? (n + 255) / 256 : (n + 127) / 128;
  int64_t best = 0;
  bool found = false;
  const int cands[2] = {pair ? 256 : 128, pair ? 224 : 112};
  for (int bn : cands) {
    const int per_cta = pair ? bn / 2 : bn;
    // the tallest box that fits (fewest loads per stage; at most 16 boxes)
    for (int r = per_cta / static_cast<int>(w); r >= 1; --r) {
      if ((w * r) % 8 != 0 || h % r != 0 || per_cta % (w * r) != 0) continue;
      if (per_cta / (w * r) > kConvMaxBoxes) break;
      const int64_t tiles = row_tiles * ((m + bn - 1) / bn);
      const int64_t waves = (tiles + units - 1) / units;
      if (!found || waves < best) {
        best = waves;
        t->pair = pair;
        t->bn = bn;
        t->rows = r;
        t->boxes = static_cast<int>(per_cta / (w * r));
        found = true;
      }
      break;
    }
  }
  return found;
}

template <int kDtype, int BN, int ST, int ST32, int ACC>
sp24_status launch_conv_pair(const CUtensorMap& ma, const GemmArgs& a, const void* x, int pairs,
                             cudaStream_t s, const ConvGeom& cg) {
  if constexpr (kDtype == SP24_BF16) {
    return launch_pair<kDtype, BN, ST, SP24_OUT_BF16, ACC, true>(ma, a, x, pairs, s, &cg);
  } else {
    if (a.out_kind == SP24_OUT_INT32)
      return launch_pair<kDtype, BN, ST32, SP24_OUT_INT32, ACC, true>(ma, a, x, pairs, s, &cg);
    if (a.out_kind == SP24_OUT_INT8)
      return launch_pair<kDtype, BN, ST, SP24_OUT_INT8, ACC, true>(ma, a, x, pairs, s, &cg);
    return launch_pair<kDtype, BN, ST, SP24_OUT_BF16, ACC, true>(ma, a, x, pairs, s, &cg);
  }
}

template <int kDtype, int BN>
sp24_status launch_conv_single(const CUtensorMap& ma, const GemmArgs& a, const void* x,
                               cudaStream_t s, const ConvGeom& cg) {
  const int el = kDtype == SP24_BF16 ? 2 : 1;
  const CUtensorMapDataType dt =
      kDtype == SP24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap mb;
  SP24_TRY(make_map_nhwc(&mb, x, dt, el, static_cast<uint64_t>(cg.c), static_cast<uint64_t>(cg.w),
                         static_cast<uint64_t>(cg.h), static_cast<uint64_t>(cg.b),
                         static_cast<uint32_t>(128 / el), static_cast<uint32_t>(cg.w),
                         static_cast<uint32_t>(cg.rows)));
  if constexpr (kDtype == SP24_BF16) {
    return launch_persistent<kDtype, BN, 4, SP24_OUT_BF16, true>(ma, mb, a, s, &cg);
  } else {
    if (a.out_kind == SP24_OUT_INT32)
      return launch_persistent<kDtype, BN, 3, SP24_OUT_INT32, true>(ma, mb, a, s, &cg);
    if (a.out_kind == SP24_OUT_INT8)
      return launch_persistent<kDtype, BN, 4, SP24_OUT_INT8, true>(ma, mb, a, s, &cg);
    return launch_persistent<kDtype, BN, 4, SP24_OUT_BF16, true>(ma, mb, a, s, &cg);
  }
}

template <int kDtype>
sp24_status conv_dispatch(const void* x, const void* vals, const GemmArgs& a, const ConvGeom& cg,
                          const ConvTile& t, cudaStream_t s) {
  const int el = kDtype == SP24_BF16 ? 2 : 1;
  const CUtensorMapDataType dt =
      kDtype == SP24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUtensorMap ma;
  SP24_TRY(make_map(&ma, vals, dt, el, static_cast<uint64_t>(a.k / 2), static_cast<uint64_t>(a.n),
                    static_cast<uint32_t>(128 / el), 128));
  if (!t.pair) {
    if (t.bn == 128) return launch_conv_single<kDtype, 128>(ma, a, x, s, cg);
    return launch_conv_single<kDtype, 112>(ma, a, x, s, cg);
  }
  int pairs = 0;
  SP24_TRY(pair_capacity(&pairs));
  const int64_t tiles = ((a.n + 255) / 256) * ((a.m + t.bn - 1) / t.bn);
  const int p = static_cast<int>(tiles < pairs ? tiles : pairs);
  if (t.bn == 256) return launch_conv_pair<kDtype, 256, 4, 3, 1>(ma, a, x, p, s, cg);
  return launch_conv_pair<kDtype, 224, 4, 4, 2>(ma, a, x, p, s, cg);
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

sp24_status sp24_conv3x3(const void* X, int64_t B, int64_t H, int64_t W, int64_t C,
                         const void* vals, const void* meta, int64_t Cout, int dtype,
                         const float* s_x, const float* s_w, int out_kind, const float* s_y,
                         void* Y, void* stream) {
  if (B < 0 || H < 0 || W < 0 || C < 0 || Cout < 0 || (dtype != SP24_BF16 && dtype != SP24_INT8))
    return SP24_ERR_ARG;
  if (dtype == SP24_BF16 && out_kind != SP24_OUT_BF16) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind != SP24_OUT_BF16 && out_kind != SP24_OUT_INT32 &&
      out_kind != SP24_OUT_INT8)
    return SP24_ERR_ARG;
  if (B == 0 || H == 0 || W == 0 || Cout == 0) return SP24_OK;
  if (C == 0) return SP24_ERR_ARG;
  if (!X || !vals || !meta || !Y) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind != SP24_OUT_INT32 && (!s_x || !s_w)) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind == SP24_OUT_INT8 && !s_y) return SP24_ERR_ARG;
  const int el = dtype == SP24_BF16 ? 2 : 1;
  if ((C * el) % 128 != 0 || Cout % 8 != 0) return SP24_ERR_ALIGN;
  if (out_kind == SP24_OUT_INT8 && dtype == SP24_INT8 && Cout % 16 != 0) return SP24_ERR_ALIGN;
  if (!aligned16(X) || !aligned16(vals) || !aligned16(meta) || !aligned16(Y) ||
      (s_w && !aligned16(s_w)))
    return SP24_ERR_ALIGN;
  const int64_t M = B * H * W, K = 9 * C;
  if (M > (int64_t(1) << 31) || K > (int64_t(1) << 31) || Cout > (int64_t(1) << 31) ||
      B > (int64_t(1) << 30))
    return SP24_ERR_UNSUPPORTED;
  SP24_TRY(check_device());
  const int kl = dtype == SP24_BF16 ? 128 : 256;
  const int kblocks = static_cast<int>((K + kl - 1) / kl);
  conv::ConvTile t;
  if (!conv::conv_tile(M, Cout, H, W, &t)) return SP24_ERR_UNSUPPORTED;
  GemmArgs a;
  a.meta = static_cast<const uint8_t*>(meta);
  a.s_x = s_x;
  a.s_w = s_w;
  a.s_y = s_y;
  a.y = Y;
  a.m = M;
  a.n = Cout;
  a.k = K;
  a.out_kind = out_kind;
  a.kblocks = kblocks;
  a.kb_per_split = kblocks;
  ConvGeom cg;
  cg.b = B;
  cg.h = H;
  cg.w = W;
  cg.c = C;
  cg.rows = t.rows;
  cg.boxes = t.boxes;
  cudaStream_t s = as_stream(stream);
  if (dtype == SP24_BF16) return conv::conv_dispatch<SP24_BF16>(X, vals, a, cg, t, s);
  return conv::conv_dispatch<SP24_INT8>(X, vals, a, cg, t, s);
}

}  // extern "C"
