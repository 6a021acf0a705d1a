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

// Threads of the persistent GEMM kernels: warp 0 producer, warp 1 MMA issuer,
// warps 2..9 epilogue; the implicit convolution adds two warps (warp 10 a
// second producer, warp 11 idle), which costs no registers: blocks are
// allocated registers in whole groups of four warps.
constexpr int kConvProducerWarp = 2 + kEpiWarps;
__host__ __device__ constexpr int gemm_threads(bool conv) { return 64 + kEpiThreads + (conv ? 64 : 0); }

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
__device__ __forceinline__ void pack_vec(const uint32_t (&r)[32], const float (&cs)[4],
                                         uint32_t (&pk)[16]) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = 16 * (q >> 1) + 4 * b + 2 * (q & 1);
      pk[4 * b + q] = pack_bf16x2(epi_value<kDtype>(r[i], cs[q]), epi_value<kDtype>(r[i + 1], cs[q]));
    }
  }
}

template <int NB>
__device__ __forceinline__ void stmatrix_vec(const uint32_t (&pk)[16], uint32_t stg, int lane) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const int tok = 8 * b + (lane & 7);
    const int chunk = (lane >> 3) ^ ((tok >> 1) & 3);
    stmatrix_x4_trans(stg + tok * 64 + chunk * 16, pk[4 * b], pk[4 * b + 1], pk[4 * b + 2],
                      pk[4 * b + 3]);
  }
}

template <int kDtype, int NB>
__device__ __forceinline__ void stage_vec(const uint32_t (&r)[32], uint32_t stg, int lane,
                                          const float (&cs)[4]) {
  uint32_t pk[16];
  pack_vec<kDtype, NB>(r, cs, pk);
  stmatrix_vec<NB>(pk, stg, lane);
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

// Stages one loaded chunk (c) of this warp and issues its TMA store.
template <int kDtype, int OUTK>
__device__ __forceinline__ void epi_store_chunk(const EpiWarp& e, const CUtensorMap* tmap_y,
                                                const CUtensorMap* tmap_y16, int c, bool half,
                                                int lane, const uint32_t (&r)[32]) {
  const int64_t t0 = e.tok0 + c * kEpiChunk;
  if (e.c0 >= e.n || t0 >= e.m) return;   // no channel of this quadrant / token of the chunk
  if (lane == 0) bulk_wait_read<0>();     // this warp's previous store read out
  __syncwarp();
  if (e.vec) {
    if (half) stage_vec<kDtype, 2>(r, smem_u32(e.stg), lane, e.cs);
    else stage_vec<kDtype, 4>(r, smem_u32(e.stg), lane, e.cs);
  } else if (e.c0 + lane < e.n) {
    if (half) stage_scalar<kDtype, OUTK, 16>(r, e.stg, lane, e.cbox, e.cs[0], e.sy);
    else stage_scalar<kDtype, OUTK, 32>(r, e.stg, lane, e.cbox, e.cs[0], e.sy);
  }
  fence_async_shared();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(half ? tmap_y16 : tmap_y, e.stg, e.c0, static_cast<int32_t>(t0));
    bulk_commit();
  }
}

// Drains this warp's chunks (grp, grp + 2, ...) of one tile.  With BN % 32 ==
// 16 the tile's last chunk holds 16 tokens and is stored through `tmap_y16`
// (16-token boxes), so no store reaches past the tile.  `release` runs once
// the warp's last tensor-memory load has completed (the accumulator may then
// be reused); all lanes call it.
//   kHoldAll = false: the next chunk's load is issued before the current
//     chunk is staged (two chunks of registers); the accumulator is released
//     after the last load, i.e. after most of the staging.  Used where a
//     second accumulator lets the next tile's MMAs run meanwhile.
//   kHoldAll = true (bf16 output through the transposing path; otherwise as
//     false): all of the warp's chunks are loaded and packed to bf16 pairs in
//     registers first and the accumulator is released before any staging, so
//     with a single accumulator the next tile's MMAs wait only for the loads.
template <int kDtype, int OUTK, int BN, bool kHoldAll, class Release>
__device__ __forceinline__ void epilogue_tile(const EpiWarp& e, const CUtensorMap* tmap_y,
                                              const CUtensorMap* tmap_y16, int grp, int lane,
                                              Release&& release) {
  static_assert(BN % 16 == 0, "tile width");
  constexpr int kChunks = (BN + kEpiChunk - 1) / kEpiChunk;
  constexpr bool kHalfTail = BN % kEpiChunk != 0;
  static_assert(kChunks >= 2, "each warp of a quadrant must own a chunk of every tile");
  constexpr int kMaxMine = (kChunks + 1) / 2;
  const int nmine = (kChunks - grp + 1) / 2;
  if (kHoldAll && OUTK == SP24_OUT_BF16 && e.vec) {
    // two chunks at a time: load, wait, pack to bf16 pairs (16 registers a
    // chunk); the accumulator is released once every chunk is packed
    uint32_t pk[kMaxMine][16];
#pragma unroll
    for (int i = 0; i < kMaxMine; i += 2) {
      uint32_t r[2][32];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = grp + 2 * (i + u);
        if (i + u < kMaxMine && i + u < nmine) epi_load(e, c, kHalfTail && c == kChunks - 1, r[u]);
      }
      tmem_ld_wait();
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int c = grp + 2 * (i + u);
        if (i + u < kMaxMine && i + u < nmine) {
          if (kHalfTail && c == kChunks - 1) pack_vec<kDtype, 2>(r[u], e.cs, pk[i + u]);
          else pack_vec<kDtype, 4>(r[u], e.cs, pk[i + u]);
        }
      }
    }
    release();
#pragma unroll
    for (int i = 0; i < kMaxMine; ++i) {
      const int c = grp + 2 * i;
      const bool half = kHalfTail && c == kChunks - 1;
      const int64_t t0 = e.tok0 + c * kEpiChunk;
      if (i < nmine && e.c0 < e.n && t0 < e.m) {
        if (lane == 0) bulk_wait_read<0>();     // this warp's previous store read out
        __syncwarp();
        if (half) stmatrix_vec<2>(pk[i], smem_u32(e.stg), lane);
        else stmatrix_vec<4>(pk[i], smem_u32(e.stg), lane);
        fence_async_shared();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(half ? tmap_y16 : tmap_y, e.stg, e.c0, static_cast<int32_t>(t0));
          bulk_commit();
        }
      }
    }
  } else {
    uint32_t r[2][32];
    if (nmine > 0) epi_load(e, grp, kHalfTail && grp == kChunks - 1, r[0]);
#pragma unroll
    for (int i = 0; i < kMaxMine; ++i) {
      if (i < nmine) {
        const int c = grp + 2 * i;
        tmem_ld_wait();   // chunk i landed (and nothing else is outstanding)
        if (i + 1 < nmine) epi_load(e, c + 2, kHalfTail && c + 2 == kChunks - 1, r[(i + 1) & 1]);
        else release();
        epi_store_chunk<kDtype, OUTK>(e, tmap_y, tmap_y16, c, kHalfTail && c == kChunks - 1, lane,
                                      r[i & 1]);
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
