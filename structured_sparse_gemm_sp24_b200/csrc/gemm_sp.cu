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
// Split-K.  When the output tiles alone cannot fill the GPU (small M: the
// weight stream is the bound), S CTAs of a thread-block cluster split the K
// blocks of one tile; their partial accumulators are summed in a fixed order
// through distributed shared memory, so the result does not depend on timing.
//
// Warp roles (128 threads): warp 0 lane 0 issues TMA, warp 1 lane 0 issues
// tcgen05 (copy + MMA), warp 2 owns the tensor-memory allocation; all four
// warps run the epilogue (tcgen05.ld of their 32 lanes -> scale / cast ->
// shared-memory transpose -> coalesced 16-byte stores of Y rows).
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

template <int kDtype, int BN, int STAGES>
struct GemmCfg {
  static constexpr int kABytes = 128 * 128;                         // A tile per stage
  static constexpr int kBHalfBytes = BN * 128;                      // one B half
  static constexpr int kMetaChunks = kDtype == SP24_BF16 ? 1 : 2;   // 2048 B each
  static constexpr int kEBytes = 2048 * kMetaChunks;
  static constexpr int kStageBytes = kABytes + 2 * kBHalfBytes + kEBytes;
  static constexpr int kLogicalK = kDtype == SP24_BF16 ? 128 : 256;  // K per stage
  static constexpr int kMmaK = kLogicalK / 4;                        // K per MMA
  static constexpr int kMetaCols = 4 * kMetaChunks;                  // TMEM columns per stage
  // accumulator columns [0, BN), two metadata buffers after it
  static constexpr int kMetaCol0 = BN;
  static constexpr int kTmemNeeded = BN + 2 * kMetaCols;
  static constexpr int kTmemCols = kTmemNeeded <= 32 ? 32
                                   : kTmemNeeded <= 64 ? 64
                                   : kTmemNeeded <= 128 ? 128
                                   : kTmemNeeded <= 256 ? 256 : 512;
  // stages are 1024-aligned: A, then the two B halves, then E
  static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
  static constexpr int kSmemBytes = STAGES * kStageStride + 1024 /*align slack*/ + 256 /*bars*/;
  static_assert(kTmemNeeded <= 512, "tensor memory overflow");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  // epilogue staging of a partial tile (fp32/int32, [BN][128]) reuses the ring
  static_assert(STAGES * kStageStride >= BN * 128 * 4, "staging does not fit");
};

// Instruction descriptor of tcgen05.mma.sp (M = 128, K-major A and B).
template <int kDtype, int BN>
__device__ __forceinline__ uint32_t make_idesc(uint32_t id2) {
  const uint32_t c_fmt = kDtype == SP24_BF16 ? 1u : 2u;  // F32 : S32
  const uint32_t ab_fmt = 1u;                             // BF16 : signed int8
  return (id2 & 3u) | (1u << 2) | (c_fmt << 4) | (ab_fmt << 7) | (ab_fmt << 10) |
         (static_cast<uint32_t>(BN >> 3) << 17) | ((128u >> 4) << 24);
}

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

template <int kDtype, int BN, int STAGES, int SPLIT>
__global__ void __launch_bounds__(128, 1)
gemm_sp_kernel(const __grid_constant__ CUtensorMap tmap_a,
               const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
  pdl_launch_dependents();
  pdl_wait_prior();
  using C = GemmCfg<kDtype, BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * C::kStageStride);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* accum_bar = empty_bar + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t split = SPLIT > 1 ? cluster_ctarank() : 0u;
  const int64_t row_tile = blockIdx.y;
  const int64_t tok_tile = blockIdx.z;
  const int kb_begin = static_cast<int>(split) * args.kb_per_split;
  int kb_end = kb_begin + args.kb_per_split;
  if (kb_end > args.kblocks) kb_end = args.kblocks;
  const int n_iters = kb_end > kb_begin ? kb_end - kb_begin : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    const int kchunks = static_cast<int>((args.k + 127) / 128);
    const uint8_t* meta_tile = args.meta + row_tile * static_cast<int64_t>(kchunks) * 2048;
    for (int i = 0; i < n_iters; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1u;
      if (!mbar_wait(&empty_bar[s], ph ^ 1u)) { *abort_flag = 1; break; }
      const int kb = kb_begin + i;
      uint8_t* st = smem + s * C::kStageStride;
      int chunks = C::kMetaChunks;
      if (kDtype == SP24_INT8 && 2 * kb + 1 >= kchunks) chunks = 1;
      mbar_arrive_expect_tx(&full_bar[s], C::kABytes + 2 * C::kBHalfBytes + 2048 * chunks);
      // A: compressed columns [kb*128B) of rows [row_tile*128, +128)
      tma_load_2d(st, &tmap_a, &full_bar[s], kb * (kDtype == SP24_BF16 ? 64 : 128),
                  static_cast<int32_t>(row_tile * 128));
      // B: logical K [kb*KL, +KL) of tokens [tok_tile*BN, +BN), two halves
      const int kx = kb * C::kLogicalK;
      const int half = C::kLogicalK / 2;
      tma_load_2d(st + C::kABytes, &tmap_b, &full_bar[s], kx,
                  static_cast<int32_t>(tok_tile * BN));
      tma_load_2d(st + C::kABytes + C::kBHalfBytes, &tmap_b, &full_bar[s], kx + half,
                  static_cast<int32_t>(tok_tile * BN));
      // E: metadata chunk(s) of this K block
      const int c0 = kb * C::kMetaChunks;
      bulk_load(st + C::kABytes + 2 * C::kBHalfBytes, meta_tile + static_cast<int64_t>(c0) * 2048,
                2048u * chunks, &full_bar[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    const int64_t k_total = args.k;
    for (int i = 0; i < n_iters; ++i) {
      const int s = i % STAGES;
      const uint32_t ph = (i / STAGES) & 1u;
      if (!mbar_wait(&full_bar[s], ph)) { *abort_flag = 1; break; }
      tc_fence_after();
      const int kb = kb_begin + i;
      uint8_t* st = smem + s * C::kStageStride;
      const uint32_t a_addr = smem_u32(st);
      const uint32_t b_addr = smem_u32(st + C::kABytes);
      const uint32_t e_addr = smem_u32(st + C::kABytes + 2 * C::kBHalfBytes);
      const uint32_t meta_col = C::kMetaCol0 + (i & 1) * C::kMetaCols;
      // MMAs that touch real K positions in this stage (the tail stage may
      // need fewer; the rest would only multiply zero fill)
      const int64_t k_left = k_total - static_cast<int64_t>(kb) * C::kLogicalK;
      int n_mma = static_cast<int>((k_left + C::kMmaK - 1) / C::kMmaK);
      n_mma = n_mma > 4 ? 4 : n_mma;
      const int chunks = kDtype == SP24_BF16 ? 1 : (n_mma > 2 ? 2 : 1);
      for (int c = 0; c < chunks; ++c) {
        // 128 rows x 16 bytes, rows contiguous: core matrices of 8 rows at 128 B
        tc_cp_128x128b(tmem_base + meta_col + 4 * c,
                       smem_desc(e_addr + 2048 * c, 128, 128, kSwizzleNone));
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (j < n_mma) {
          const uint64_t a_desc = smem_desc(a_addr + 32 * j, 0, 1024, kSwizzle128B);
          const uint64_t b_desc =
              smem_desc(b_addr + (j >> 1) * C::kBHalfBytes + 64 * (j & 1), 0, 1024, kSwizzle128B);
          const uint32_t accumulate = (i > 0 || j > 0) ? 1u : 0u;
          if constexpr (kDtype == SP24_BF16) {
            tc_mma_sp(tmem_base, a_desc, b_desc, tmem_base + meta_col + (j & ~1),
                      make_idesc<kDtype, BN>(j & 1), accumulate);
          } else {
            tc_mma_sp_i8(tmem_base, a_desc, b_desc, tmem_base + meta_col + 2 * j,
                         make_idesc<kDtype, BN>(0), accumulate);
          }
        }
      }
      tc_commit(&empty_bar[s]);   // frees the stage once these MMAs are done
    }
    tc_commit(accum_bar);         // accumulator complete
  }
  __syncwarp();

  // ---------------------------------------------------------------- epilogue
  if (n_iters > 0 && !mbar_wait(accum_bar, 0)) *abort_flag = 1;
  tc_fence_after();
  __syncthreads();
  const bool ok = *abort_flag == 0;   // uniform across the CTA

  const int row_local = threadIdx.x;  // TMEM lane = output channel within the tile
  const uint32_t lane_addr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
  // staging buffer reuses the (now idle) pipeline ring: [BN][128] 32-bit
  uint32_t* stage32 = reinterpret_cast<uint32_t*>(smem);

  // 1) accumulator -> shared memory, token-major (raw 32-bit accumulators)
  if (ok && n_iters > 0) {
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 16) {
      uint32_t r[16];
      tmem_ld16(lane_addr + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) stage32[(c0 + j) * 128 + row_local] = r[j];
    }
  } else {
    for (int c0 = 0; c0 < BN; ++c0) stage32[c0 * 128 + row_local] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (SPLIT > 1) cluster_sync();   // all partials visible cluster-wide

  // 2) reduce over the split CTAs (fixed rank order), scale / cast, store.
  //    CTA `split` owns tokens [split*BN/SPLIT, (split+1)*BN/SPLIT).
  constexpr int kTokPerCta = BN / SPLIT;
  const int tok0 = static_cast<int>(split) * kTokPerCta;
  // work item = (token, group of 4 channels); 32 groups per token
  const float sx = (kDtype == SP24_INT8 && args.out_kind != SP24_OUT_INT32) ? *args.s_x : 1.0f;
  const float sy = (kDtype == SP24_INT8 && args.out_kind == SP24_OUT_INT8) ? *args.s_y : 1.0f;
  for (int item = threadIdx.x; item < kTokPerCta * 32; item += 128) {
    const int t = tok0 + item / 32;
    const int g = item % 32;
    const int64_t m_idx = tok_tile * BN + t;
    const int64_t n0 = row_tile * 128 + 4 * g;
    if (m_idx >= args.m || n0 >= args.n) continue;
    const uint32_t off = smem_u32(stage32 + t * 128 + 4 * g);
    uint4 acc;
    if constexpr (SPLIT > 1) {
      acc = ld_cluster_v4(map_peer(off, 0));
      for (int q = 1; q < SPLIT; ++q) {
        const uint4 p = ld_cluster_v4(map_peer(off, q));
        if constexpr (kDtype == SP24_BF16) {
          acc.x = __float_as_uint(__fadd_rn(__uint_as_float(acc.x), __uint_as_float(p.x)));
          acc.y = __float_as_uint(__fadd_rn(__uint_as_float(acc.y), __uint_as_float(p.y)));
          acc.z = __float_as_uint(__fadd_rn(__uint_as_float(acc.z), __uint_as_float(p.z)));
          acc.w = __float_as_uint(__fadd_rn(__uint_as_float(acc.w), __uint_as_float(p.w)));
        } else {
          acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
        }
      }
    } else {
      acc = *reinterpret_cast<const uint4*>(stage32 + t * 128 + 4 * g);
    }
    const uint32_t a4[4] = {acc.x, acc.y, acc.z, acc.w};
    if constexpr (kDtype == SP24_BF16) {
      __nv_bfloat16* y = static_cast<__nv_bfloat16*>(args.y) + m_idx * args.n + n0;
      __nv_bfloat162 lo = __floats2bfloat162_rn(__uint_as_float(a4[0]), __uint_as_float(a4[1]));
      __nv_bfloat162 hi = __floats2bfloat162_rn(__uint_as_float(a4[2]), __uint_as_float(a4[3]));
      uint2 o;
      o.x = *reinterpret_cast<uint32_t*>(&lo);
      o.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(y) = o;
    } else if (args.out_kind == SP24_OUT_INT32) {
      int32_t* y = static_cast<int32_t*>(args.y) + m_idx * args.n + n0;
      *reinterpret_cast<uint4*>(y) = acc;
    } else {
      float f[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float c = __fmul_rn(sx, __ldg(args.s_w + n0 + j));
        f[j] = __fmul_rn(__int2float_rn(static_cast<int32_t>(a4[j])), c);
      }
      if (args.out_kind == SP24_OUT_BF16) {
        __nv_bfloat16* y = static_cast<__nv_bfloat16*>(args.y) + m_idx * args.n + n0;
        __nv_bfloat162 lo = __floats2bfloat162_rn(f[0], f[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(f[2], f[3]);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&lo);
        o.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(y) = o;
      } else {
        uint32_t packed = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          int q = __float2int_rn(__fdiv_rn(f[j], sy));
          q = q > 127 ? 127 : (q < -127 ? -127 : q);
          packed |= (static_cast<uint32_t>(q) & 0xFFu) << (8 * j);
        }
        int8_t* y = static_cast<int8_t*>(args.y) + m_idx * args.n + n0;
        *reinterpret_cast<uint32_t*>(y) = packed;
      }
    }
  }
  __syncwarp();
  if constexpr (SPLIT > 1) cluster_sync();   // peers finished reading our partials

  if (!ok) settle_ns(20000);   // let copies already in flight land
  __syncthreads();
  if (warp == 2) tmem_dealloc(tmem_base, C::kTmemCols);
}

}  // namespace sp24

#include "gemm_epilogue.cuh"
#include "gemm_persistent.cuh"
#include "gemm_pair.cuh"

namespace sp24 {

// ----------------------------------------------------------------- host side
namespace {

template <int kDtype, int BN, int STAGES, int SPLIT>
sp24_status launch_gemm_cfg(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a,
                            cudaStream_t s) {
  using C = GemmCfg<kDtype, BN, STAGES>;
  auto kern = gemm_sp_kernel<kDtype, BN, STAGES, SPLIT>;
  static uint64_t attr_set = 0;   // one bit per device (devices 0..63)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
    attr_set |= bit;
  }
  const int64_t row_tiles = (a.n + 127) / 128;
  const int64_t tok_tiles = (a.m + BN - 1) / BN;
  if (row_tiles > 65535 || tok_tiles > 65535) return SP24_ERR_UNSUPPORTED;
  return launch_kernel(kern, dim3(SPLIT, static_cast<unsigned>(row_tiles),
                                  static_cast<unsigned>(tok_tiles)),
                       dim3(128), C::kSmemBytes, s, SPLIT, ma, mb, a);
}


template <int kDtype, int BN, int STAGES, int OUTK>
sp24_status launch_persistent(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g,
                              cudaStream_t s) {
  using C = PersistCfg<kDtype, BN, STAGES, OUTK>;
  auto kern = gemm_sp_persistent<kDtype, BN, STAGES, OUTK>;
  static uint64_t attr_set = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
    attr_set |= bit;
  }
  const CUtensorMapDataType ydt = OUTK == SP24_OUT_INT32 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                  : OUTK == SP24_OUT_INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                          : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int y_box = epi_box(g.n);
  CUtensorMap my;
  SP24_TRY(make_map(&my, g.y, ydt, C::kOutBytes, static_cast<uint64_t>(g.n),
                    static_cast<uint64_t>(g.m), static_cast<uint32_t>(y_box), kEpiChunk,
                    epi_vec<OUTK>(g.n) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE));
  PersistArgs a;
  a.meta = g.meta;
  a.s_x = g.s_x;
  a.s_w = g.s_w;
  a.s_y = g.s_y;
  a.m = g.m;
  a.n = g.n;
  a.k = g.k;
  a.kblocks = g.kblocks;
  a.row_tiles = static_cast<int>((g.n + 127) / 128);
  a.tok_tiles = static_cast<int>((g.m + BN - 1) / BN);
  // raster group: as many weight row tiles as fit ~24 MB of compressed weights
  const int64_t row_tile_bytes = 128 * (g.k / 2) * (kDtype == SP24_BF16 ? 2 : 1);
  int64_t gr = (int64_t(24) << 20) / (row_tile_bytes > 0 ? row_tile_bytes : 1);
  gr = gr < 1 ? 1 : (gr > a.row_tiles ? a.row_tiles : gr);
  a.group_rows = static_cast<int>(gr);
  a.y_box = y_box;
  const int64_t ntiles = static_cast<int64_t>(a.row_tiles) * a.tok_tiles;
  if (ntiles > 0x7FFFFFFF) return SP24_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(ntiles < sm_count() ? ntiles : sm_count());
  return launch_kernel(kern, dim3(grid), dim3(64 + kEpiThreads), C::kSmemBytes, s, 1, ma, mb, my,
                       a);
}


template <int kDtype, int BN, int STAGES, int OUTK, int ACC>
sp24_status launch_pair(const CUtensorMap& ma, const GemmArgs& g, const void* x, int pairs,
                        cudaStream_t s) {
  using C = PairCfg<kDtype, BN, STAGES, OUTK, ACC>;
  auto kern = gemm_sp_pair<kDtype, BN, STAGES, OUTK, ACC>;
  static uint64_t attr_set = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_set & bit)) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
    attr_set |= bit;
  }
  const int el = kDtype == SP24_BF16 ? 2 : 1;
  const CUtensorMapDataType dt =
      kDtype == SP24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  // B: each CTA loads BN/2 token rows
  CUtensorMap mb;
  SP24_TRY(make_map(&mb, x, dt, el, static_cast<uint64_t>(g.k), static_cast<uint64_t>(g.m),
                    static_cast<uint32_t>(128 / el), static_cast<uint32_t>(C::kHalfN)));
  // E: metadata chunks as rows of 256 bytes (8 rows per 2048-byte chunk)
  const int64_t kchunks = (g.k + 127) / 128;
  const int64_t rt128 = (g.n + 127) / 128;
  CUtensorMap me;
  SP24_TRY(make_map(&me, g.meta, CU_TENSOR_MAP_DATA_TYPE_UINT64, 8, 32,
                    static_cast<uint64_t>(rt128 * kchunks * 8), 32,
                    static_cast<uint32_t>(8 * C::kMetaChunks), CU_TENSOR_MAP_SWIZZLE_NONE));
  const CUtensorMapDataType ydt = OUTK == SP24_OUT_INT32 ? CU_TENSOR_MAP_DATA_TYPE_INT32
                                  : OUTK == SP24_OUT_INT8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                          : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int y_box = epi_box(g.n);
  const CUtensorMapSwizzle yswz =
      epi_vec<OUTK>(g.n) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUtensorMap my, my16;
  SP24_TRY(make_map(&my, g.y, ydt, C::kOutBytes, static_cast<uint64_t>(g.n),
                    static_cast<uint64_t>(g.m), static_cast<uint32_t>(y_box), kEpiChunk, yswz));
  // tiles of 16 (mod 32) tokens store their last chunk with 16-token boxes
  if (BN % kEpiChunk != 0) {
    SP24_TRY(make_map(&my16, g.y, ydt, C::kOutBytes, static_cast<uint64_t>(g.n),
                      static_cast<uint64_t>(g.m), static_cast<uint32_t>(y_box), 16, yswz));
  } else {
    my16 = my;
  }
  PersistArgs a;
  a.meta = g.meta;
  a.s_x = g.s_x;
  a.s_w = g.s_w;
  a.s_y = g.s_y;
  a.m = g.m;
  a.n = g.n;
  a.k = g.k;
  a.kblocks = g.kblocks;
  a.row_tiles = static_cast<int>((g.n + 255) / 256);
  a.tok_tiles = static_cast<int>((g.m + BN - 1) / BN);
  const int64_t row_tile_bytes = 256 * (g.k / 2) * el;
  int64_t gr = (int64_t(24) << 20) / (row_tile_bytes > 0 ? row_tile_bytes : 1);
  gr = gr < 1 ? 1 : (gr > a.row_tiles ? a.row_tiles : gr);
  a.group_rows = static_cast<int>(gr);
  a.y_box = y_box;
  const int64_t ntiles = static_cast<int64_t>(a.row_tiles) * a.tok_tiles;
  if (ntiles > 0x7FFFFFFF) return SP24_ERR_UNSUPPORTED;
  if (pairs < 1 || pairs > ntiles) return SP24_ERR_ARG;   // the plan sizes the grid
  return launch_kernel(kern, dim3(2 * pairs), dim3(64 + kEpiThreads), C::kSmemBytes, s, 2, ma,
                       mb, me, my, my16, a);
}

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

// SP24_SPLITK = 1 | 2 | 4 | 8: K slices of the split-K kernel (tuning
// override; 0 = choose by shape).
int split_override() {
  const char* e = std::getenv("SP24_SPLITK");
  if (!e) return 0;
  const int v = std::atoi(e);
  return (v == 1 || v == 2 || v == 4 || v == 8) ? v : 0;
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

// CTA pairs (clusters of 2) that can be resident at once.  A cluster lives in
// one GPC, so a GPC with an odd number of SMs leaves one out and the count can
// be below SMs / 2; the persistent pair kernels launch exactly this many pairs
// so that no pair waits for another to finish.  Every pair variant holds one
// CTA per SM, so one query (cached per device) serves them all.
sp24_status pair_capacity(int* out) {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  if (cache[dev & 63] > 0) {
    *out = cache[dev & 63];
    return SP24_OK;
  }
  using C = PairCfg<SP24_BF16, 256, 4, SP24_OUT_BF16, 1>;
  auto kern = gemm_sp_pair<SP24_BF16, 256, 4, SP24_OUT_BF16, 1>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute", e);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sm_count() / 2), 1, 1);
  cfg.blockDim = dim3(64 + kEpiThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
  if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveClusters", e);
  if (n < 1) return SP24_ERR_UNSUPPORTED;
  cache[dev & 63] = n;
  *out = n;
  return SP24_OK;
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
    case kPair256:   // one accumulator: the whole epilogue is exposed
      return waves(prow * ((m + 255) / 256), pairs) * (0.50 * kb + 2.5);
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
  int64_t ctas;        // CTAs launched
  int cluster;         // CTAs per cluster
  int tile_tokens;     // tokens (rows of X and Y) per output tile
  int tile_channels;   // output channels (rows of W) per output tile
};

// The launch plan.  At least 128 tokens and enough 128 x 128 tiles for half
// the SMs: a persistent kernel, the variant with the lowest estimated time (or
// the SP24_GEMM_IMPL override).  Otherwise (few tokens or few tiles): the
// split-K kernel, BN from the token count and K split as far as all CTAs still
// fit one wave (SP24_SPLITK overrides the split).
sp24_status make_plan(int64_t m, int64_t n, int kblocks, Plan* p) {
  const int sms = sm_count();
  const int64_t row_tiles = (n + 127) / 128;
  const int forced = impl_override();
  if (forced != kSplitK && m >= 128 && row_tiles * ((m + 127) / 128) >= sms / 2) {
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
  // one CTA per SM fits (the rings take most of shared memory), so the K
  // split stops where the CTAs would exceed one wave: measured on B200 for
  // M = 16..256 decode shapes, a second wave costs more than the longer K
  // loop of a smaller split (e.g. M = 16, 11008 x 4096: split 1 on 86 SMs
  // 20.5 us, split 4 on 344 CTAs 29 us)
  int split = 1;
  while (split < 8 && base * split * 2 <= sms && kblocks >= 4 * split) split *= 2;
  const int so = split_override();
  if (so > 0 && so <= kblocks) split = so;
  p->impl = kSplitK;
  p->bn = bn;
  p->split = split;
  p->ctas = base * split;
  p->cluster = split;
  p->tile_tokens = bn;
  p->tile_channels = 128;
  return SP24_OK;
}

// CTA-pair kernel for every output kind; ST = ring stages (ST32 with int32
// output, whose staging is twice the size).
template <int kDtype, int BN, int ST, int ST32, int ACC>
sp24_status launch_pair_out(const CUtensorMap& ma, const GemmArgs& a, const void* x, int pairs,
                            cudaStream_t s) {
  if constexpr (kDtype == SP24_BF16) {
    return launch_pair<kDtype, BN, ST, SP24_OUT_BF16, ACC>(ma, a, x, pairs, s);
  } else {
    if (a.out_kind == SP24_OUT_INT32)
      return launch_pair<kDtype, BN, ST32, SP24_OUT_INT32, ACC>(ma, a, x, pairs, s);
    if (a.out_kind == SP24_OUT_INT8)
      return launch_pair<kDtype, BN, ST, SP24_OUT_INT8, ACC>(ma, a, x, pairs, s);
    return launch_pair<kDtype, BN, ST, SP24_OUT_BF16, ACC>(ma, a, x, pairs, s);
  }
}

template <int kDtype>
sp24_status dispatch(const void* x, const void* vals, GemmArgs a, cudaStream_t s) {
  Plan p;
  SP24_TRY(make_plan(a.m, a.n, a.kblocks, &p));
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
    switch (split) {                                                                      \
      case 1: return launch_gemm_cfg<kDtype, BN_, ST_, 1>(ma, mb, a, s);                  \
      case 2: return launch_gemm_cfg<kDtype, BN_, ST_, 2>(ma, mb, a, s);                  \
      case 4: return launch_gemm_cfg<kDtype, BN_, ST_, 4>(ma, mb, a, s);                  \
      default: return launch_gemm_cfg<kDtype, BN_, ST_, 8>(ma, mb, a, s);                 \
    }                                                                                     \
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
  SP24_TRY(make_plan(M, N, static_cast<int>((K + kl - 1) / kl), &p));
  std::memset(plan, 0, sizeof(*plan));
  std::snprintf(plan->kernel, sizeof(plan->kernel), "%s", impl_name(p.impl));
  plan->tile_tokens = p.tile_tokens;
  plan->tile_channels = p.tile_channels;
  plan->split_k = p.split;
  plan->ctas = p.ctas;
  plan->cluster = p.cluster;
  return SP24_OK;
}
