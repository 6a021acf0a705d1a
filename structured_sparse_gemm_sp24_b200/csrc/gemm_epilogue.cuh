// Epilogue shared by the persistent GEMM kernels (single-SM and CTA-pair).
// Included by gemm_sp.cu.
//
// Eight epilogue warps: warp w reaches tensor-memory lane quadrant w % 4 (32
// output channels of the 128-row tile), and the two warps of a quadrant split
// the tile's 32-token chunks between them (group 0: chunks 0, 2, 4, ...;
// group 1: chunks 1, 3, 5, ...).  Each warp works alone -- no barrier with
// other warps -- on a [32 tokens][32 channels] box per chunk:
//   tcgen05.ld -> cast / dequantise in registers -> its own shared-memory
//   staging box -> its own TMA tensor store (clipped at the M / N edges).
// The next chunk's tensor-memory load is issued before the current chunk is
// staged, so its latency overlaps the staging and the store.
//
// Y is [M tokens][N channels] with channels contiguous, while a thread's
// accumulators run along tokens, so staging is a transpose.  For bf16 output
// (N >= 32) it is done by stmatrix .trans on the mma fragment layout that the
// 16x256b tensor-memory load produces: four instructions per warp and chunk,
// into a box stored with the 64-byte swizzle so that the eight 16-byte rows
// of each 8x8 matrix fall in distinct banks.  int32 and int8 outputs (and bf16
// with N < 32) take one store per token from the 32x32b load, where a thread
// owns one channel and the warp writes whole box rows.
#pragma once

namespace sp24 {

constexpr int kEpiChunk = 32;            // tokens (accumulator columns) per chunk
constexpr int kEpiWarps = 8;             // two per lane quadrant
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kEpiBox = 32;              // channels per warp store box

template <int OUTK>
struct EpiOut {
  static constexpr int kBytes = OUTK == SP24_OUT_INT32 ? 4 : (OUTK == SP24_OUT_INT8 ? 1 : 2);
  static constexpr int kWarpBytes = kEpiChunk * kEpiBox * kBytes;   // one staging box
  static constexpr int kStagingBytes = kEpiWarps * kWarpBytes;
};

// Box width in channels (min(32, N)) and whether the transposing bf16 path is
// used; the store tensor map must be encoded to match (64-byte swizzle iff vec).
inline int epi_box(int64_t n) { return static_cast<int>(n < kEpiBox ? n : kEpiBox); }
template <int OUTK>
inline bool epi_vec(int64_t n) { return OUTK == SP24_OUT_BF16 && n >= kEpiBox; }

struct EpiWarp {
  uint32_t tmem;          // this warp's lane quadrant + accumulator column 0 of the tile
  uint8_t* stg;           // this warp's staging box
  int64_t tok0;           // first token of the tile
  int64_t m, n;           // problem sizes
  int c0;                 // first output channel of this warp's quadrant
  int cbox;               // store box width in channels
  bool vec;               // transposing bf16 path
  float cs[4];            // int8 dequant factor of the channels this thread stages
  float sy;               // int8 requant scale
};

template <int kDtype>
__device__ __forceinline__ float epi_value(uint32_t acc, float cscale) {
  if constexpr (kDtype == SP24_BF16) return __uint_as_float(acc);
  return __fmul_rn(__int2float_rn(static_cast<int32_t>(acc)), cscale);
}

// Transposing path.  Register 16h + 4b + 2s + u holds channel 16h + 8s + lane/4
// and token 8b + 2(lane%4) + u (from two 16x256b loads at lane offsets 0 and
// 16), so the pair u = 0, 1 is one b32 of the 8x8 matrix (channels 8(2h+s) ..,
// tokens 8b ..).  Thread `lane` addresses token row 8b + lane%8 of matrix
// lane/8 for stmatrix; the box row is 64 bytes and its 16-byte chunk index is
// XORed with bits 1-2 of the row (64-byte swizzle).
template <int kDtype, int NB>
__device__ __forceinline__ void stage_vec(const uint32_t (&r)[32], uint32_t stg, int lane,
                                          const float (&cs)[4]) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 16 * (q >> 1) + 4 * b + 2 * (q & 1);
      p[q] = pack_bf16x2(epi_value<kDtype>(r[i], cs[q]), epi_value<kDtype>(r[i + 1], cs[q]));
    }
    const int tok = 8 * b + (lane & 7);
    const int chunk = (lane >> 3) ^ ((tok >> 1) & 3);
    stmatrix_x4_trans(stg + tok * 64 + chunk * 16, p[0], p[1], p[2], p[3]);
  }
}

// One-channel-per-thread path (thread `lane` owns channel c0 + lane), NT tokens.
template <int kDtype, int OUTK, int NT>
__device__ __forceinline__ void stage_scalar(const uint32_t (&r)[32], uint8_t* stg, int lane,
                                             int cbox, float cscale, float sy) {
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int e = t * cbox + lane;
    if constexpr (kDtype == SP24_BF16) {
      reinterpret_cast<__nv_bfloat16*>(stg)[e] = __float2bfloat16_rn(__uint_as_float(r[t]));
    } else if constexpr (OUTK == SP24_OUT_INT32) {
      reinterpret_cast<uint32_t*>(stg)[e] = r[t];
    } else {
      const float f = epi_value<kDtype>(r[t], cscale);
      if constexpr (OUTK == SP24_OUT_BF16) {
        reinterpret_cast<__nv_bfloat16*>(stg)[e] = __float2bfloat16_rn(f);
      } else {
        int qv = __float2int_rn(__fdiv_rn(f, sy));
        qv = qv > 127 ? 127 : (qv < -127 ? -127 : qv);
        reinterpret_cast<int8_t*>(stg)[e] = static_cast<int8_t>(qv);
      }
    }
  }
}

__device__ __forceinline__ void epi_load(const EpiWarp& e, int chunk, bool half,
                                         uint32_t (&r)[32]) {
  const uint32_t ta = e.tmem + static_cast<uint32_t>(chunk * kEpiChunk);
  if (e.vec) {
    if (half) {
      tmem_ld_16x256b_x2<0>(ta, r);
      tmem_ld_16x256b_x2<1>(ta + (16u << 16), r);
    } else {
      tmem_ld_16x256b_x4<0>(ta, r);
      tmem_ld_16x256b_x4<1>(ta + (16u << 16), r);
    }
  } else if (half) {
    tmem_ld16_into(ta, r);
  } else {
    tmem_ld32(ta, r);
  }
}

// Drains this warp's chunks (grp, grp + 2, ...) of one tile.  With BN % 32 ==
// 16 the tile's last chunk holds 16 tokens and is stored through `tmap_y16`
// (16-token boxes), so no store reaches past the tile.  `release` runs once
// the warp's last tensor-memory load has completed (the accumulator may then
// be reused); all lanes call it.
template <int kDtype, int OUTK, int BN, class Release>
__device__ __forceinline__ void epilogue_tile(const EpiWarp& e, const CUtensorMap* tmap_y,
                                              const CUtensorMap* tmap_y16, int grp, int lane,
                                              Release&& release) {
  static_assert(BN % 16 == 0, "tile width");
  constexpr int kChunks = (BN + kEpiChunk - 1) / kEpiChunk;
  constexpr bool kHalfTail = BN % kEpiChunk != 0;
  static_assert(kChunks >= 2, "each warp of a quadrant must own a chunk of every tile");
  constexpr int kMaxMine = (kChunks + 1) / 2;
  const int nmine = (kChunks - grp + 1) / 2;
  const bool live = e.c0 < e.n;   // some channel of this quadrant exists
  uint32_t r[2][32];
  if (nmine > 0) epi_load(e, grp, kHalfTail && grp == kChunks - 1, r[0]);
#pragma unroll
  for (int i = 0; i < kMaxMine; ++i) {
    if (i < nmine) {
      const int c = grp + 2 * i;
      const bool half = kHalfTail && c == kChunks - 1;
      tmem_ld_wait();   // chunk i landed (and nothing else is outstanding)
      if (i + 1 < nmine) epi_load(e, c + 2, kHalfTail && c + 2 == kChunks - 1, r[(i + 1) & 1]);
      else release();
      const int64_t t0 = e.tok0 + c * kEpiChunk;
      if (live && t0 < e.m) {
        if (lane == 0) bulk_wait_read<0>();         // this warp's previous store read out
        __syncwarp();
        if (e.vec) {
          if (half) stage_vec<kDtype, 2>(r[i & 1], smem_u32(e.stg), lane, e.cs);
          else stage_vec<kDtype, 4>(r[i & 1], smem_u32(e.stg), lane, e.cs);
        } else if (e.c0 + lane < e.n) {
          if (half) stage_scalar<kDtype, OUTK, 16>(r[i & 1], e.stg, lane, e.cbox, e.cs[0], e.sy);
          else stage_scalar<kDtype, OUTK, 32>(r[i & 1], e.stg, lane, e.cbox, e.cs[0], e.sy);
        }
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(half ? tmap_y16 : tmap_y, e.stg, e.c0, static_cast<int32_t>(t0));
          bulk_commit();
        }
      }
    }
  }
}

// Per-tile dequant factors: the vector path stages channels c0 + lane/4 +
// 8q (q = 0..3), the scalar path channel c0 + lane.
template <int kDtype, int OUTK>
__device__ __forceinline__ void epi_scales(EpiWarp& e, int lane, const float* s_w, float sx) {
  if constexpr (kDtype == SP24_INT8 && OUTK != SP24_OUT_INT32) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t c = e.c0 + (e.vec ? (lane >> 2) + 8 * q : lane);
      e.cs[q] = c < e.n ? __fmul_rn(sx, __ldg(s_w + c)) : 0.0f;
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) e.cs[q] = 0.0f;
  }
}

}  // namespace sp24
