// libsp24: sparse GEMM Y = X * W'^T on the 5th-generation tensor cores
// (tcgen05.mma.sp), for bf16 (fp32 accumulate) and int8 (int32 accumulate).
//
// [Orin ch.7] "Chapter 7: 2:4 Structured Sparsity" 2.1 Step 3: the sparse
// tensor core multiplies only the kept weights, each with the activation its
// 2-bit position selects; [Sparse-accel forum] (oeforum.com): INT8 x 2:4.
//
// Operand roles.  The sparse operand of tcgen05.mma.sp is A (the MMA's M
// side), so the kernel computes one 128 (output channels) x BN (tokens) tile
// of Y^T = W' * X^T per CTA:
//   A = compressed W tile: 128 rows x 128 bytes per stage (bf16: 64 values =
//       128 logical K; int8: 128 values = 256 logical K), TMA, 128B swizzle;
//   B = X tile: BN rows x 256 bytes per stage as two 128B-swizzled halves;
//   E = metadata chunk(s) (2048 bytes per 128 logical K), one bulk copy, then
//       tcgen05.cp into tensor memory, where tcgen05.mma.sp reads it;
//   D = fp32 / int32 accumulator in tensor memory: lane = output channel,
//       column = token.
// Each stage issues 4 MMAs (K = 32 for kind::f16, 64 for kind::i8); both
// advance A by 32 bytes and B by 64 bytes inside the swizzle atoms.
//
// Kernels: gemm_splitk.cuh (split-K), gemm_persistent.cuh (single-SM
// persistent), gemm_pair.cuh (CTA-pair persistent), each with its launch;
// gemm_epilogue.cuh (epilogue of both persistent kernels).  This file holds
// the launch plan, the dispatch and the C entry points.

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "sp24_device.cuh"
#include "sp24_host.h"
#include "tma_host.h"

namespace sp24 {

struct GemmArgs {
  const uint8_t* meta;
  const float* s_x;
  const float* s_w;
  const float* s_y;
  void* y;
  int64_t m, n, k;
  int kblocks;        // stages over the whole K
  int kb_per_split;   // stages per split CTA
  int out_kind;
};

}  // namespace sp24

#include "gemm_splitk.cuh"
#include "gemm_epilogue.cuh"
#include "gemm_persistent.cuh"
#include "gemm_pair.cuh"

namespace sp24 {

// ----------------------------------------------------------------- host side
namespace {

// Which kernel to use: SP24_GEMM_IMPL = pair256 | pair240 | pair224 | pair192 |
// pair128 | single | splitk (tuning override; default chooses by problem size).
enum Impl : int { kSplitK = 0, kPair256 = 1, kPair128 = 2, kSingle = 3, kPair224 = 4,
                  kPair192 = 5, kPair240 = 6 };

int impl_override() {
  const char* e = std::getenv("SP24_GEMM_IMPL");
  if (!e) return -1;
  if (std::strcmp(e, "pair256") == 0) return kPair256;
  if (std::strcmp(e, "pair128") == 0) return kPair128;
  if (std::strcmp(e, "single") == 0) return kSingle;
  if (std::strcmp(e, "pair224") == 0) return kPair224;
  if (std::strcmp(e, "pair192") == 0) return kPair192;
  if (std::strcmp(e, "pair240") == 0) return kPair240;
  if (std::strcmp(e, "splitk") == 0) return kSplitK;
  return -1;
}

// SP24_SPLITK = 1..8: K slices of the split-K kernel (tuning override; 0 =
// choose by shape).
int split_override() {
  const char* e = std::getenv("SP24_SPLITK");
  if (!e) return 0;
  const int v = std::atoi(e);
  return (v >= 1 && v <= 8) ? v : 0;
}

const char* impl_name(int impl) {
  switch (impl) {
    case kPair256: return "pair256";
    case kPair240: return "pair240";
    case kPair224: return "pair224";
    case kPair192: return "pair192";
    case kPair128: return "pair128";
    case kSingle: return "single";
    default: return "splitk";
  }
}

int pair_tokens(int impl) {
  switch (impl) {
    case kPair256: return 256;
    case kPair240: return 240;
    case kPair224: return 224;
    case kPair192: return 192;
    default: return 128;
  }
}

// Estimated run time (us, B200 under load) of a persistent variant: waves of
// output tiles over the SMs (resident pairs) x per-tile time, i.e. k-blocks x
// the measured cost of one k-block plus the part of the epilogue the variant
// cannot overlap with the next tile.  Used only to rank the variants.
double est_time(int impl, int64_t m, int64_t n, int kblocks, int sms, int pairs) {
  const auto waves = [](int64_t tiles, int64_t units) {
    return static_cast<double>((tiles + units - 1) / units);
  };
  const double kb = kblocks;
  const int64_t prow = (n + 255) / 256;
  switch (impl) {
    case kPair256:   // one accumulator: the next tile waits for the epilogue's
                     // tensor-memory loads (~0.8 us a tile, measured)
      return waves(prow * ((m + 255) / 256), pairs) * (0.50 * kb + 0.8);
    case kPair240:   // two accumulators: only the last drain is exposed
      return waves(prow * ((m + 239) / 240), pairs) * std::max(0.50 * kb, 1.5) + 2.0;
    case kPair224:
      return waves(prow * ((m + 223) / 224), pairs) * std::max(0.50 * kb, 1.4) + 2.0;
    default:         // 128 x 128 single-SM tile, two accumulators
      return waves(((n + 127) / 128) * ((m + 127) / 128), sms) * std::max(0.48 * kb, 1.6);
  }
}

struct Plan {
  int impl;            // Impl
  int bn;              // split-K kernel: tokens per tile
  int split;           // split-K kernel: K slices (= cluster size)
  bool small_ring;     // split-K kernel: the ring that lets several CTAs share an SM
  int64_t ctas;        // CTAs launched
  int cluster;         // CTAs per cluster
  int tile_tokens;     // tokens (rows of X and Y) per output tile
  int tile_channels;   // output channels (rows of W) per output tile
};

// The launch plan.  At least 128 tokens and at least one 128 x 128 tile per
// SM: a persistent kernel, the variant with the lowest estimated time (or the
// SP24_GEMM_IMPL override).  Otherwise (few tokens or less than one wave of
// tiles): the split-K kernel, BN from the token count and K split as far as
// all CTAs still fit one wave (SP24_SPLITK overrides the split).  Measured on
// B200: M = 128 x 11008 x 4096 (86 tiles) takes 22.5 us split-K, 24.6 us on
// the persistent kernel.
// Split-K rings: the full ring (one CTA per SM) and a small one with which
// several split CTAs share an SM (so that a split spreads a few row tiles
// over every SM without a second wave).  Shared memory per SM on sm_100 is
// 228 KiB, of which each resident CTA also takes 1 KiB.  With either ring
// the CTAs that fit an SM by shared memory need at most 512 tensor-memory
// columns together (16 tokens: 3 x 32; 32: 4 x 64; 64: 3 x 128; 128:
// 2 x 256), so no CTA's allocation ever waits on another's.
constexpr int kSmemPerSm = 228 * 1024;
constexpr int small_ring_stages(int bn) { return bn == 16 ? 3 : 2; }

template <int kDtype>
int small_ring_smem(int bn) {
  switch (bn) {
    case 16: return GemmCfg<kDtype, 16, small_ring_stages(16)>::kSmemBytes;
    case 32: return GemmCfg<kDtype, 32, small_ring_stages(32)>::kSmemBytes;
    case 64: return GemmCfg<kDtype, 64, small_ring_stages(64)>::kSmemBytes;
    default: return GemmCfg<kDtype, 128, small_ring_stages(128)>::kSmemBytes;
  }
}

int small_ring_ctas_per_sm(int dtype, int bn) {
  const int smem = dtype == SP24_BF16 ? small_ring_smem<SP24_BF16>(bn)
                                      : small_ring_smem<SP24_INT8>(bn);
  return kSmemPerSm / (smem + 1024);
}

sp24_status make_plan(int64_t m, int64_t n, int kblocks, int dtype, Plan* p) {
  const int sms = sm_count();
  const int64_t row_tiles = (n + 127) / 128;
  const int forced = impl_override();
  // (an SP24_GEMM_IMPL override applies from half a wave of tiles, as the
  // kernel-family tests expect)
  const int64_t tiles128 = row_tiles * ((m + 127) / 128);
  if (forced != kSplitK && m >= 128 && tiles128 >= (forced >= 0 ? sms / 2 : sms)) {
    int pairs = 0;
    SP24_TRY(pair_capacity(&pairs));
    int impl = forced;
    if (impl < 0) {
      impl = kSingle;   // pair tiles need both dimensions to fill them
      if (m >= 256 && n >= 256) {
        double best = est_time(kSingle, m, n, kblocks, sms, pairs);
        for (int c : {kPair256, kPair240, kPair224}) {
          const double t = est_time(c, m, n, kblocks, sms, pairs);
          if (t < best) {
            best = t;
            impl = c;
          }
        }
      }
    }
    p->impl = impl;
    p->bn = 128;
    p->split = 1;
    p->small_ring = false;
    if (impl == kSingle) {
      const int64_t tiles = row_tiles * ((m + 127) / 128);
      p->ctas = tiles < sms ? tiles : sms;
      p->cluster = 1;
      p->tile_tokens = 128;
      p->tile_channels = 128;
    } else {
      const int tok = pair_tokens(impl);
      const int64_t tiles = ((n + 255) / 256) * ((m + tok - 1) / tok);
      p->ctas = 2 * (tiles < pairs ? tiles : pairs);
      p->cluster = 2;
      p->tile_tokens = tok;
      p->tile_channels = 256;
    }
    return SP24_OK;
  }
  const int bn = m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : 128;
  const int64_t base = row_tiles * ((m + bn - 1) / bn);
  // The split.  A stage's sparse MMAs take about the same time whatever the
  // token count (measured on B200: ~0.44 us per 128-channel x 128-K stage at
  // 16 tokens, ~0.5 us at 256), so at few tokens the kernel is bound by the
  // stages the busiest SM runs: ceil(CTAs / SMs) x stages per CTA.  The plan
  // takes the split among 1, 2, 4, 8 (at least 4 stages per CTA) that
  // minimises it, the fewer CTAs on a tie; more than one CTA per SM takes
  // the small ring.  E.g. M = 16, 11008 x 4096 (86 row tiles, 32 stages):
  // split 1 on 86 SMs runs 32 stages on the busiest SM, split 4 (344 CTAs,
  // 3 per SM) 24 -- 9.8 against 13.9 us a launch back to back.  Splits of 3,
  // 5, 6 and 7 run correctly (SP24_SPLITK) but measured no better: at 3 CTAs
  // per SM a GPC holds fewer 5-CTA clusters than the 86 tiles need
  // (cudaOccupancyMaxActiveClusters: 82), and the second wave costs more
  // than the shorter K loop saves.
  int split = 1;
  int64_t best = -1;
  const int cap = small_ring_ctas_per_sm(dtype, bn);
  for (int sp = 1; sp <= 8; sp *= 2) {
    if (sp > 1 && kblocks < 4 * sp) break;
    const int64_t per_sm = (base * sp + sms - 1) / sms;
    if (sp > 1 && per_sm > cap) break;
    const int64_t cost = per_sm * ((kblocks + sp - 1) / sp);
    if (best < 0 || cost < best) {
      best = cost;
      split = sp;
    }
  }
  const int so = split_override();
  if (so > 0 && so <= kblocks) split = so;
  p->impl = kSplitK;
  p->bn = bn;
  p->split = split;
  p->small_ring = base * split > sms;
  p->ctas = base * split;
  p->cluster = split;
  p->tile_tokens = bn;
  p->tile_channels = 128;
  return SP24_OK;
}

template <int kDtype, int BN, int ST>
sp24_status launch_split(int split, const CUtensorMap& ma, const CUtensorMap& mb,
                         const GemmArgs& a, cudaStream_t s) {
  switch (split) {
    case 1: return launch_gemm_cfg<kDtype, BN, ST, 1>(ma, mb, a, s);
    case 2: return launch_gemm_cfg<kDtype, BN, ST, 2>(ma, mb, a, s);
    case 3: return launch_gemm_cfg<kDtype, BN, ST, 3>(ma, mb, a, s);
    case 4: return launch_gemm_cfg<kDtype, BN, ST, 4>(ma, mb, a, s);
    case 5: return launch_gemm_cfg<kDtype, BN, ST, 5>(ma, mb, a, s);
    case 6: return launch_gemm_cfg<kDtype, BN, ST, 6>(ma, mb, a, s);
    case 7: return launch_gemm_cfg<kDtype, BN, ST, 7>(ma, mb, a, s);
    default: return launch_gemm_cfg<kDtype, BN, ST, 8>(ma, mb, a, s);
  }
}

template <int kDtype>
sp24_status dispatch(const void* x, const void* vals, GemmArgs a, cudaStream_t s) {
  Plan p;
  SP24_TRY(make_plan(a.m, a.n, a.kblocks, kDtype, &p));
  a.kb_per_split = (a.kblocks + p.split - 1) / p.split;
  const int bn = p.bn;
  const int el = kDtype == SP24_BF16 ? 2 : 1;
  const CUtensorMapDataType dt =
      kDtype == SP24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const uint32_t box_cols = 128 / el;
  CUtensorMap ma, mb;
  SP24_TRY(make_map(&ma, vals, dt, el, static_cast<uint64_t>(a.k / 2),
                    static_cast<uint64_t>(a.n), box_cols, 128));
  const int pairs = static_cast<int>(p.ctas / 2);
  switch (p.impl) {
    case kPair256: return launch_pair_out<kDtype, 256, 4, 3, 1>(ma, a, x, pairs, s);
    case kPair240: return launch_pair_out<kDtype, 240, 4, 3, 2>(ma, a, x, pairs, s);
    case kPair224: return launch_pair_out<kDtype, 224, 4, 4, 2>(ma, a, x, pairs, s);
    case kPair192: return launch_pair_out<kDtype, 192, 4, 4, 2>(ma, a, x, pairs, s);
    case kPair128:
      if constexpr (kDtype == SP24_BF16) {
        return launch_pair<kDtype, 128, 6, SP24_OUT_BF16, 2>(ma, a, x, pairs, s);
      } else {
        if (a.out_kind == SP24_OUT_INT32)
          return launch_pair<kDtype, 128, 5, SP24_OUT_INT32, 2>(ma, a, x, pairs, s);
        if (a.out_kind == SP24_OUT_INT8)
          return launch_pair<kDtype, 128, 6, SP24_OUT_INT8, 2>(ma, a, x, pairs, s);
        return launch_pair<kDtype, 128, 5, SP24_OUT_BF16, 2>(ma, a, x, pairs, s);
      }
    default: break;
  }
  SP24_TRY(make_map(&mb, x, dt, el, static_cast<uint64_t>(a.k), static_cast<uint64_t>(a.m),
                    box_cols, static_cast<uint32_t>(bn)));
  if (p.impl == kSingle) {
    if constexpr (kDtype == SP24_BF16) {
      return launch_persistent<kDtype, 128, 4, SP24_OUT_BF16>(ma, mb, a, s);
    } else {
      if (a.out_kind == SP24_OUT_INT32) return launch_persistent<kDtype, 128, 3, SP24_OUT_INT32>(ma, mb, a, s);
      if (a.out_kind == SP24_OUT_INT8) return launch_persistent<kDtype, 128, 4, SP24_OUT_INT8>(ma, mb, a, s);
      return launch_persistent<kDtype, 128, 4, SP24_OUT_BF16>(ma, mb, a, s);
    }
  }
  const int split = p.split;

#define SP24_GEMM_CASE(BN_, ST_)                                                          \
  if (bn == BN_) {                                                                        \
    constexpr int kSm = small_ring_stages(BN_);                                           \
    if (p.small_ring) return launch_split<kDtype, BN_, kSm>(split, ma, mb, a, s);          \
    return launch_split<kDtype, BN_, ST_>(split, ma, mb, a, s);                             \
  }
  SP24_GEMM_CASE(16, 8)
  SP24_GEMM_CASE(32, 8)
  SP24_GEMM_CASE(64, 6)
  SP24_GEMM_CASE(128, 4)
#undef SP24_GEMM_CASE
  return SP24_ERR_UNSUPPORTED;
}

}  // namespace
}  // namespace sp24

using namespace sp24;

extern "C" sp24_status sp24_gemm(const void* X, int64_t M, int64_t K, const void* vals,
                                 const void* meta, int64_t N, int dtype, const float* s_x,
                                 const float* s_w, int out_kind, const float* s_y, void* Y,
                                 void* stream) {
  if (M < 0 || N < 0 || K < 0 || (dtype != SP24_BF16 && dtype != SP24_INT8)) return SP24_ERR_ARG;
  if (dtype == SP24_BF16 && out_kind != SP24_OUT_BF16) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind != SP24_OUT_BF16 && out_kind != SP24_OUT_INT32 &&
      out_kind != SP24_OUT_INT8)
    return SP24_ERR_ARG;
  if (M == 0 || N == 0) return SP24_OK;
  if (!X || !vals || !meta || !Y) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind != SP24_OUT_INT32 && (!s_x || !s_w)) return SP24_ERR_ARG;
  if (dtype == SP24_INT8 && out_kind == SP24_OUT_INT8 && !s_y) return SP24_ERR_ARG;
  if (K < 16 || N % 8 != 0 || K % (dtype == SP24_BF16 ? 16 : 32) != 0) return SP24_ERR_ALIGN;
  if (out_kind == SP24_OUT_INT8 && dtype == SP24_INT8 && N % 16 != 0) return SP24_ERR_ALIGN;
  if (!aligned16(X) || !aligned16(vals) || !aligned16(meta) || !aligned16(Y) ||
      (s_w && !aligned16(s_w)))
    return SP24_ERR_ALIGN;
  if (K > (int64_t(1) << 31) || M > (int64_t(1) << 31) || N > (int64_t(1) << 31))
    return SP24_ERR_UNSUPPORTED;
  SP24_TRY(check_device());
  if (!get_encoder()) return cuda_fail("cudaGetDriverEntryPoint", "cuTensorMapEncodeTiled");
  GemmArgs a;
  a.meta = static_cast<const uint8_t*>(meta);
  a.s_x = s_x;
  a.s_w = s_w;
  a.s_y = s_y;
  a.y = Y;
  a.m = M;
  a.n = N;
  a.k = K;
  a.out_kind = out_kind;
  const int kl = dtype == SP24_BF16 ? 128 : 256;
  a.kblocks = static_cast<int>((K + kl - 1) / kl);
  a.kb_per_split = a.kblocks;
  if (dtype == SP24_BF16) return dispatch<SP24_BF16>(X, vals, a, as_stream(stream));
  return dispatch<SP24_INT8>(X, vals, a, as_stream(stream));
}

extern "C" sp24_status sp24_gemm_plan(int64_t M, int64_t N, int64_t K, int dtype,
                                      sp24_gemm_plan_t* plan) {
  if (!plan || M < 1 || N < 1 || K < 16 || (dtype != SP24_BF16 && dtype != SP24_INT8))
    return SP24_ERR_ARG;
  if (K > (int64_t(1) << 31) || M > (int64_t(1) << 31) || N > (int64_t(1) << 31))
    return SP24_ERR_UNSUPPORTED;
  SP24_TRY(check_device());
  const int kl = dtype == SP24_BF16 ? 128 : 256;
  Plan p;
  SP24_TRY(make_plan(M, N, static_cast<int>((K + kl - 1) / kl), dtype, &p));
  std::memset(plan, 0, sizeof(*plan));
  std::snprintf(plan->kernel, sizeof(plan->kernel), "%s", impl_name(p.impl));
  plan->tile_tokens = p.tile_tokens;
  plan->tile_channels = p.tile_channels;
  plan->split_k = p.split;
  plan->ctas = p.ctas;
  plan->cluster = p.cluster;
  return SP24_OK;
}
