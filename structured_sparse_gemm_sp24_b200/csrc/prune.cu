// libsp24: Wanda column norms, N:4 pruning, compression (bf16 / int8) into the
// tcgen05.mma.sp operand layout, INT8 calibration scales and quantisation.
//
// All of these are HBM-bound streaming kernels: 16-byte vector loads of W,
// one pass over the data, grid sized in multiples of the SM count.
//
// Sources: [Wanda-2:4] "Structured Pruning: 2:4 sparse inference with the
// Wanda algorithm" sections 1.3, 2.1, 2.2; [Orin ch.7] "Chapter 7: 2:4
// Structured Sparsity" section 2.1 (worked 1x4 example: rule, compressed data
// stream, 2-bit metadata) and 6.1 (every 1x4 block must be valid);
// [Ampere-sparsity] NVIDIA x Tencent article, Figure 1 (values + index
// metadata), Figure 4 (progressive 25 % -> 50 %), "PTQ and QAT" (99.99 %
// coverage scale).
#include <cuda.h>

#include <mutex>

#include "sp24_device.cuh"
#include "sp24_host.h"
#include "tma_host.h"

namespace sp24 {

// ------------------------------------------------------------- scoring keys
// Magnitude order of a finite bf16 equals the unsigned order of its low 15
// bits, so magnitude scores compare exactly as integers (and -0 == +0).
__device__ __forceinline__ uint32_t mag_key(uint32_t bits16) { return bits16 & 0x7FFFu; }

__device__ __forceinline__ double bf16_to_double(uint32_t bits16) {
  return static_cast<double>(__uint_as_float(bits16 << 16));
}

// Rank rule for one group of 4: position p is kept iff fewer than n_keep
// others beat it; for p < q, p beats q when s_p >= s_q (ties to the lower
// index), otherwise q beats p.  Returns the keep nibble (bit p = kept).
template <typename S>
__device__ __forceinline__ uint32_t keep_nibble(S s0, S s1, S s2, S s3, int n_keep) {
  int b0 = 0, b1 = 0, b2 = 0, b3 = 0;
  if (s0 >= s1) ++b1; else ++b0;
  if (s0 >= s2) ++b2; else ++b0;
  if (s0 >= s3) ++b3; else ++b0;
  if (s1 >= s2) ++b2; else ++b1;
  if (s1 >= s3) ++b3; else ++b1;
  if (s2 >= s3) ++b3; else ++b2;
  return static_cast<uint32_t>(b0 < n_keep) | (static_cast<uint32_t>(b1 < n_keep) << 1) |
         (static_cast<uint32_t>(b2 < n_keep) << 2) | (static_cast<uint32_t>(b3 < n_keep) << 3);
}

// Keep mask byte for 8 consecutive weights of one row (two groups): low
// nibble = first group.  `w` holds the 8 bf16 patterns, `in` the mask_in byte
// (0xFF when absent), `nrm` the 8 column norms (Wanda only).
template <bool kWanda>
__device__ __forceinline__ uint32_t mask_byte(const uint4& w, uint32_t in, const double* nrm,
                                              int n_keep) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t out = 0;
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    uint32_t b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t word = words[2 * g + i / 2];
      const uint32_t bits = (i & 1) ? (word >> 16) : (word & 0xFFFFu);
      const bool live = (in >> (4 * g + i)) & 1u;
      b[i] = live ? bits : 0u;
    }
    uint32_t nib;
    if constexpr (kWanda) {
      double s[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) s[i] = __dmul_rn(fabs(bf16_to_double(b[i])), nrm[4 * g + i]);
      nib = keep_nibble(s[0], s[1], s[2], s[3], n_keep);
    } else {
      nib = keep_nibble(mag_key(b[0]), mag_key(b[1]), mag_key(b[2]), mag_key(b[3]), n_keep);
    }
    out |= nib << (4 * g);
  }
  return out;
}

// ------------------------------------------------ fast magnitude selection
// Augmented keys K_p = (|w_p| bits << 2) | (3 - p) of one group (4 bf16 in two
// 32-bit words): all distinct, and K_q > K_p exactly when q beats p under the
// rank rule (larger magnitude; equal magnitudes go to the lower index).  A
// position dropped by mask_in scores magnitude 0 and keeps its index order.
// The kept set is then the n_keep largest keys.
template <bool kLive>
__device__ __forceinline__ uint32_t keep_nibble_mag(uint32_t w0, uint32_t w1, uint32_t live,
                                                    int n_keep) {
  uint32_t k0 = ((w0 << 2) & 0x1FFFCu) | 3u;
  uint32_t k1 = ((w0 >> 14) & 0x1FFFCu) | 2u;
  uint32_t k2 = ((w1 << 2) & 0x1FFFCu) | 1u;
  uint32_t k3 = ((w1 >> 14) & 0x1FFFCu);
  if constexpr (kLive) {
    k0 = (live & 1u) ? k0 : 3u;
    k1 = (live & 2u) ? k1 : 2u;
    k2 = (live & 4u) ? k2 : 1u;
    k3 = (live & 8u) ? k3 : 0u;
  }
  const uint32_t a = max(k0, k1), b = min(k0, k1), c = max(k2, k3), d = min(k2, k3);
  if (n_keep == 2) {
    const uint32_t t1 = max(a, c);
    const uint32_t t2 = max(min(a, c), max(b, d));
    return (1u << (~t1 & 3u)) | (1u << (~t2 & 3u));
  }
  const uint32_t t4 = min(b, d);   // n_keep == 3: drop the smallest
  return 0xFu ^ (1u << (~t4 & 3u));
}

// Positions (lo < hi) of the two largest augmented keys of a group (see
// keep_nibble_mag), with integer min/max only.
template <bool kLive>
__device__ __forceinline__ void top2_positions_mag(uint32_t w0, uint32_t w1, uint32_t live,
                                                   uint32_t& lo, uint32_t& hi) {
  uint32_t k0 = ((w0 << 2) & 0x1FFFCu) | 3u;
  uint32_t k1 = ((w0 >> 14) & 0x1FFFCu) | 2u;
  uint32_t k2 = ((w1 << 2) & 0x1FFFCu) | 1u;
  uint32_t k3 = ((w1 >> 14) & 0x1FFFCu);
  if constexpr (kLive) {
    k0 = (live & 1u) ? k0 : 3u;
    k1 = (live & 2u) ? k1 : 2u;
    k2 = (live & 4u) ? k2 : 1u;
    k3 = (live & 8u) ? k3 : 0u;
  }
  const uint32_t a = max(k0, k1), b = min(k0, k1), c = max(k2, k3), d = min(k2, k3);
  const uint32_t p1 = ~max(a, c) & 3u;                     // 3 - (t & 3)
  const uint32_t p2 = ~max(min(a, c), max(b, d)) & 3u;
  lo = min(p1, p2);
  hi = max(p1, p2);
}

// Metadata code (lo | hi << 2) of a keep nibble from a 16-entry table; nibbles
// without exactly two bits set map to positions (0, 1) and are flagged.
constexpr uint64_t kNibbleCode = 0x444E4DC449844444ull;   // indices 3,5,6,9,10,12 valid
constexpr uint32_t kNibbleValid = 0x1668u;
__device__ __forceinline__ uint32_t nibble_code(uint32_t nib, uint32_t& bad) {
  bad |= ((kNibbleValid >> nib) & 1u) ^ 1u;
  return static_cast<uint32_t>(kNibbleCode >> (4u * nib)) & 0xFu;
}

// Gathers the kept bf16 pair of a group with one byte permute: low half =
// position lo, high half = position hi.
__device__ __forceinline__ uint32_t gather_pair(uint32_t w0, uint32_t w1, uint32_t lo,
                                                uint32_t hi) {
  return __byte_perm(w0, w1, 0x1010u + 0x22u * lo + 0x2200u * hi);
}

// -------------------------------------------------------------- a1 colnorm
// Block per 64 columns.  Each pass stages a [128 tokens][64 columns] bf16 tile
// in shared memory with every 16-byte load in flight, then threads 0..63 add
// the squares of their column sequentially in token order (float64, one
// rounding per addition; the square of a bf16 value is exact).
__global__ void __launch_bounds__(256) colnorm_kernel(const uint16_t* __restrict__ xc,
                                                      int64_t mc, int64_t k,
                                                      double* __restrict__ norms) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ __align__(16) uint16_t tile[128][64];
  const int64_t col0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int cvalid = static_cast<int>(k - col0 < 64 ? k - col0 : 64);   // multiple of 8
  double acc = 0.0;
  for (int64_t t0 = 0; t0 < mc; t0 += 128) {
    const int rows = static_cast<int>(mc - t0 < 128 ? mc - t0 : 128);
    // 128 x 8 16-byte pieces, four per thread, all loads issued before the stores
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = threadIdx.x + u * 256;
      const int r = i >> 3, c8 = (i & 7) * 8;
      if (r < rows && c8 < cvalid)
        v[u] = __ldg(reinterpret_cast<const uint4*>(xc + (t0 + r) * k + col0 + c8));
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = threadIdx.x + u * 256;
      const int r = i >> 3, c8 = (i & 7) * 8;
      if (r < rows && c8 < cvalid) *reinterpret_cast<uint4*>(&tile[r][c8]) = v[u];
    }
    __syncthreads();
    if (threadIdx.x < cvalid) {
      for (int r = 0; r < rows; ++r) {
        const double x = bf16_to_double(tile[r][threadIdx.x]);
        acc = __dadd_rn(acc, __dmul_rn(x, x));
      }
    }
    __syncthreads();
  }
  if (threadIdx.x < cvalid) norms[col0 + threadIdx.x] = __dsqrt_rn(acc);
}

// ------------------------------------------------------------ a4 compress
// Metadata operand layout (per 128-row x 128-K chunk, 2048 bytes; chunks
// ordered [row tile][K block]).  Source byte = (row m, byte bb of the chunk's
// 16 metadata bytes per row), covering groups 2bb, 2bb+1 of the chunk.
//   int8 (tcgen05 kind::i8): row-major, offset = 16*m + bb.
//   bf16 (kind::f16): tensor-memory lane = (m%8) + 8*((bb%4)/2) + 16*(m/16);
//        within the lane, 32-bit word j = bb/4 feeds MMA j (32 K-positions);
//        rows m%16 < 8 fill the low half-word and rows m%16 >= 8 the high one;
//        offset = 16*lane + 4*j + 2*((m/8)%2) + (bb%2).
// Nibble order inside a byte is the same as in the canonical layout.
template <int kDtype>
__device__ __forceinline__ uint32_t meta_offset(uint32_t m, uint32_t bb) {
  if constexpr (kDtype == SP24_INT8) {
    return 16u * m + bb;
  } else {
    const uint32_t lane = (m & 7u) + 8u * ((bb & 3u) >> 1) + 16u * (m >> 4);
    return 16u * lane + 4u * (bb >> 2) + 2u * ((m >> 3) & 1u) + (bb & 1u);
  }
}

// Kept positions of a nibble with exactly two bits set -> (lo | hi << 2).
// Any other nibble is a pattern error; it is recorded and encoded as (0, 1).
__device__ __forceinline__ uint32_t meta_nibble(uint32_t keep, uint32_t& bad) {
  const uint32_t lo = __ffs(keep) - 1u;
  const uint32_t hi = 31u - __clz(keep);
  const bool ok = __popc(keep) == 2;
  bad |= ok ? 0u : 1u;
  return ok ? (lo | (hi << 2)) : 0x4u;
}

template <int kDtype>
struct CompressOut;

// ------------------------------------------- a2..a4 streaming chunk kernel
// One persistent CTA per SM walks 128-row x 128-K chunks of W.  Thread 0
// keeps kStreamStages chunks in flight with TMA loads (the W chunk plus, as
// needed, the chunk's mask bytes, the 128 Wanda column norms and the 128
// per-row INT8 scales); the 1024 threads then work from shared memory: thread
// t takes vector t % 16 (8 consecutive K-positions) of chunk rows t/16 + 64*j,
// j = 0..1, so a warp reads two rows of 256 contiguous bytes.
//   kPrune: compute the keep mask (magnitude / Wanda, n_keep of 4) from W,
//           with dropped mask_in positions scoring 0; else read the mask.
//   kVals:  kValsNone   -> write the keep mask only (sp24_prune);
//           kValsBF16/INT8 -> also write values and the metadata chunk.
// The metadata chunk and the mask bytes of a chunk are assembled in shared
// memory and written with 16-byte stores.
enum { kValsNone = 0, kValsBF16 = 1, kValsINT8 = 2 };

constexpr int kStreamStages = 2;   // two CTAs per SM each keep two chunks in flight
constexpr int kStreamThreads = 512;
constexpr int kStreamRows = 128 / (kStreamThreads / 16);   // chunk rows per thread (4)
constexpr int kWTile = 128 * 256;          // 128 rows x 128 bf16
constexpr int kMTile = 128 * 16;           // 128 rows x 16 mask bytes
constexpr int kNTile = 128 * 8;            // 128 float64 norms
constexpr int kSTile = 128 * 4;            // 128 float32 row scales
constexpr int kStreamStage = kWTile + kMTile + kNTile + kSTile;   // multiple of 128
constexpr int kStreamSmem = kStreamStages * kStreamStage + 4 * 2048 + 256 + 1024;
constexpr int kXcTile = 128 * 256;   // fused Wanda norms: 128 tokens x 128 columns of Xc
constexpr int kStreamSmemFused = kStreamSmem + kXcTile;
constexpr int kProgExtra = 2 * 2048;   // progressive: staging of the first-stage mask

struct StreamArgs {
  int64_t n, k;
  int kblocks;                 // chunks along K
  int nchunks;                 // row tiles * kblocks
  int n_keep;
  int mask_tma;                // the chunk's mask bytes come with the TMA stage
  const uint8_t* mask_direct;  // else read from here (NULL: no mask / mask_in)
  uint8_t* mask_out;           // NULL: not written
  uint8_t* mask1_out;          // progressive: first-stage (3 of 4) mask, NULL: not written
  void* vals;
  uint8_t* meta;
  // Wanda with the column norms computed in the kernel (xc != NULL): each CTA
  // forms the norms of its chunk's 128 columns from Xc [mc][k]; CTAs of row
  // tile 0 also store them to norms_out
  const uint16_t* xc;
  int64_t mc;
  double* norms_out;
};

//   kProg: progressive pruning in one pass ([Ampere-sparsity] Figure 4): the
//          first-stage mask keeps 3 of 4, the second keeps 2 of 4 of the weights
//          the first stage kept (dropped ones score 0); the second mask drives
//          the values and metadata.  kPrune must be set and kMaskIn clear.
template <bool kPrune, bool kWanda, int kVals, bool kMaskIn, bool kProg = false>
__global__ void __launch_bounds__(kStreamThreads, 1)
stream_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_mask,
              const __grid_constant__ CUtensorMap tm_norm, const __grid_constant__ CUtensorMap tm_sw,
              const StreamArgs a) {
  pdl_launch_dependents();
  pdl_wait_prior();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* meta_buf = smem + kStreamStages * kStreamStage;     // 2 x 2048
  uint8_t* mout_buf = meta_buf + 2 * 2048;                     // 2 x 2048
  uint8_t* mout1_buf = mout_buf + 2 * 2048;                    // 2 x 2048 (kProg only)
  uint64_t* full = reinterpret_cast<uint64_t*>(mout_buf + 2 * 2048 + (kProg ? kProgExtra : 0));
  static_assert(!kProg || (kPrune && !kMaskIn), "progressive pruning computes its own masks");

  const int tid = threadIdx.x;
  const uint32_t bb = tid & 15u;              // vector within a chunk row
  const uint32_t m0 = tid >> 4;               // first chunk row (0..31)
  const int64_t kvec = a.k / 8;
  const int nmine = a.nchunks > static_cast<int>(blockIdx.x)
                        ? (a.nchunks - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                        : 0;
  const bool use_mask_tile = a.mask_tma != 0;
  const bool fused_norms = kWanda && a.xc != nullptr;
  const uint32_t stage_tx = kWTile + (use_mask_tile ? kMTile : 0) +
                            ((kWanda && !fused_norms) ? kNTile : 0) +
                            (kVals == kValsINT8 ? kSTile : 0);

  if (tid == 0) {
    for (int st = 0; st < kStreamStages; ++st) mbar_init(&full[st], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int i) {
    const int c = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    const int rt = c / a.kblocks, kb = c - rt * a.kblocks;
    const int st = i % kStreamStages;
    uint8_t* sb = smem + st * kStreamStage;
    mbar_arrive_expect_tx(&full[st], stage_tx);
    tma_load_2d(sb, &tm_w, &full[st], kb * 128, rt * 128);
    if (use_mask_tile) tma_load_2d(sb + kWTile, &tm_mask, &full[st], kb * 16, rt * 128);
    if (kWanda && !fused_norms) tma_load_1d(sb + kWTile + kMTile, &tm_norm, &full[st], kb * 128);
    if constexpr (kVals == kValsINT8)
      tma_load_1d(sb + kWTile + kMTile + kNTile, &tm_sw, &full[st], rt * 128);
  };
  if (tid == 0) {
    prefetch_tmap(&tm_w);
    for (int i = 0; i < nmine && i < kStreamStages; ++i) issue(i);
  }

  uint32_t bad = 0;
  for (int i = 0; i < nmine; ++i) {
    const int c = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    const int rt = c / a.kblocks, kb = c - rt * a.kblocks;
    const int st = i % kStreamStages;
    const uint8_t* sb = smem + st * kStreamStage;
    const int64_t kv = static_cast<int64_t>(kb) * 16 + bb;
    uint8_t* mb = meta_buf + (i & 1) * 2048;
    uint8_t* ob = mout_buf + (i & 1) * 2048;
    uint8_t* ob1 = mout1_buf + (i & 1) * 2048;
    double nrm[8];
    if constexpr (kWanda) {
      if (fused_norms) {
        // (formed before waiting for the chunk: they need only Xc, so its
        // loads overlap the W chunk's TMA)
        // column norms of this chunk, in the stage's norm slot (TMA does not
        // write it in this mode): Xc is staged 128 tokens at a time with
        // every 16-byte load in flight; threads 0..127 then add the squares
        // of their column in token order (float64, one rounding per product
        // and per addition), then sqrt
        // 256 bytes past the stage barriers (16-byte aligned), in the kXcTile
        // bytes a fused launch adds to the dynamic shared memory
        uint16_t(*xt)[128] = reinterpret_cast<uint16_t(*)[128]>(full + 32);
        const int64_t col0 = static_cast<int64_t>(kb) * 128;
        const int cvalid = static_cast<int>(a.k - col0 < 128 ? a.k - col0 : 128);   // % 8 == 0
        double acc = 0.0;
        for (int64_t t0 = 0; t0 < a.mc; t0 += 128) {
          const int rows = static_cast<int>(a.mc - t0 < 128 ? a.mc - t0 : 128);
          uint4 v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {   // 128 rows x 16 pieces of 8 columns
            const int q = tid + u * kStreamThreads;
            const int r = q >> 4, c8 = (q & 15) * 8;
            if (r < rows && c8 < cvalid)
              v[u] = __ldg(reinterpret_cast<const uint4*>(a.xc + (t0 + r) * a.k + col0 + c8));
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int q = tid + u * kStreamThreads;
            const int r = q >> 4, c8 = (q & 15) * 8;
            if (r < rows && c8 < cvalid) *reinterpret_cast<uint4*>(&xt[r][c8]) = v[u];
          }
          __syncthreads();
          if (tid < cvalid) {
            for (int r = 0; r < rows; ++r) {
              const double x = bf16_to_double(xt[r][tid]);
              acc = __dadd_rn(acc, __dmul_rn(x, x));
            }
          }
          __syncthreads();
        }
        if (tid < 128) {
          const double nv = __dsqrt_rn(acc);
          reinterpret_cast<double*>(const_cast<uint8_t*>(sb) + kWTile + kMTile)[tid] = nv;
          if (rt == 0 && tid < cvalid) a.norms_out[col0 + tid] = nv;
        }
        __syncthreads();
      }
    }
    const bool ready = mbar_wait(&full[st], (i / kStreamStages) & 1u);
    const bool kv_ok = kv < kvec && ready;
    double zero_sc[8];   // progressive Wanda: the score of a zero weight, 0 * n_j
    if constexpr (kWanda) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        nrm[e] = reinterpret_cast<const double*>(sb + kWTile + kMTile)[bb * 8 + e];
        if constexpr (kProg) zero_sc[e] = __dmul_rn(0.0, nrm[e]);
      }
    }
    // per-thread bases: chunk row m0 + 32 j is +8192 bytes of the W tile,
    // +512 bytes of the mask tile, of the metadata chunk (both layouts) and
    // of the mask staging, and +32 j * kvec vectors in global memory
    const uint8_t* wrow = sb + m0 * 256 + bb * 16;
    const uint8_t* mrow = sb + kWTile + m0 * 16 + bb;
    const float* srow = reinterpret_cast<const float*>(sb + kWTile + kMTile + kNTile) + m0;
    const uint32_t moff = kVals == kValsINT8 ? meta_offset<SP24_INT8>(m0, bb)
                                             : meta_offset<SP24_BF16>(m0, bb);
    const int64_t row0 = static_cast<int64_t>(rt) * 128 + m0;
    const int64_t vi0 = row0 * kvec + kv;
#pragma unroll
    for (int j = 0; j < kStreamRows; ++j) {
      const bool ok = kv_ok && row0 + 32 * j < a.n;
      const int64_t vi = vi0 + static_cast<int64_t>(32 * j) * kvec;
      uint32_t meta_byte = 0x44u;             // padding: positions (0, 1)
      uint32_t keep = 0;
      if (ok) {
        const uint4 q = *reinterpret_cast<const uint4*>(wrow + 8192 * j);
        uint32_t mbyte = 0xFFu;
        if (!kPrune || kMaskIn) {
          if (use_mask_tile) {
            mbyte = mrow[512 * j];
          } else {
            mbyte = a.mask_direct[vi];
          }
        }
        uint32_t lo0, hi0, lo1, hi1;
        if constexpr (kProg) {
          // stage 1 keeps 3 of 4; stage 2 keeps 2 of 4 of what stage 1 kept
          uint32_t k3;
          if constexpr (kWanda) {
            // the products |w| * n_j once; stage 2 scores a dropped position
            // as a zero weight (0 * n_j, as mask_byte with mask_in does)
            const uint32_t words[4] = {q.x, q.y, q.z, q.w};
            double sc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t bits = (e & 1) ? (words[e / 2] >> 16) : (words[e / 2] & 0xFFFFu);
              sc[e] = __dmul_rn(fabs(bf16_to_double(bits)), nrm[e]);
            }
            k3 = keep_nibble(sc[0], sc[1], sc[2], sc[3], 3) |
                 (keep_nibble(sc[4], sc[5], sc[6], sc[7], 3) << 4);
#pragma unroll
            for (int e = 0; e < 8; ++e) sc[e] = ((k3 >> e) & 1u) ? sc[e] : zero_sc[e];
            keep = keep_nibble(sc[0], sc[1], sc[2], sc[3], 2) |
                   (keep_nibble(sc[4], sc[5], sc[6], sc[7], 2) << 4);
          } else {
            k3 = keep_nibble_mag<false>(q.x, q.y, 0xFu, 3) |
                 (keep_nibble_mag<false>(q.z, q.w, 0xFu, 3) << 4);
            keep = keep_nibble_mag<true>(q.x, q.y, k3 & 15u, 2) |
                   (keep_nibble_mag<true>(q.z, q.w, k3 >> 4, 2) << 4);
          }
          if (a.mask1_out) ob1[m0 * 16 + bb + 512 * j] = static_cast<uint8_t>(k3);
          if constexpr (kVals != kValsNone) {
            uint32_t badv = 0;
            const uint32_t c0 = nibble_code(keep & 15u, badv);
            const uint32_t c1 = nibble_code(keep >> 4, badv);
            lo0 = c0 & 3u; hi0 = c0 >> 2; lo1 = c1 & 3u; hi1 = c1 >> 2;
          }
        } else if constexpr (kPrune && !kWanda && kVals != kValsNone) {
          top2_positions_mag<kMaskIn>(q.x, q.y, mbyte & 15u, lo0, hi0);
          top2_positions_mag<kMaskIn>(q.z, q.w, mbyte >> 4, lo1, hi1);
          if (a.mask_out) keep = (1u << lo0) | (1u << hi0) | (((1u << lo1) | (1u << hi1)) << 4);
        } else {
          if constexpr (kPrune && kWanda) {
            keep = mask_byte<true>(q, mbyte, nrm, a.n_keep);
          } else if constexpr (kPrune) {
            keep = keep_nibble_mag<kMaskIn>(q.x, q.y, mbyte & 15u, a.n_keep) |
                   (keep_nibble_mag<kMaskIn>(q.z, q.w, mbyte >> 4, a.n_keep) << 4);
          } else {
            keep = mbyte;
          }
          if constexpr (kVals != kValsNone) {
            uint32_t badv = 0;
            const uint32_t c0 = nibble_code(keep & 15u, badv);
            const uint32_t c1 = nibble_code(keep >> 4, badv);
            if (!kPrune) bad |= badv;
            lo0 = c0 & 3u; hi0 = c0 >> 2; lo1 = c1 & 3u; hi1 = c1 >> 2;
          }
        }
        if constexpr (kVals != kValsNone) {
          meta_byte = lo0 | (hi0 << 2) | (lo1 << 4) | (hi1 << 6);
          const uint32_t p0 = gather_pair(q.x, q.y, lo0, hi0);
          const uint32_t p1 = gather_pair(q.z, q.w, lo1, hi1);
          if constexpr (kVals == kValsBF16) {
            __stcs(reinterpret_cast<uint2*>(a.vals) + vi, make_uint2(p0, p1));
          } else {
            const float sc = srow[32 * j];
            const float xs[4] = {__uint_as_float(p0 << 16), __uint_as_float(p0 & 0xFFFF0000u),
                                 __uint_as_float(p1 << 16), __uint_as_float(p1 & 0xFFFF0000u)};
            uint32_t packed = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              int qv = __float2int_rn(__fdiv_rn(xs[e], sc));
              qv = qv > 127 ? 127 : (qv < -127 ? -127 : qv);
              packed |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * e);
            }
            __stcs(reinterpret_cast<unsigned int*>(a.vals) + vi, packed);
          }
        }
      }
      if constexpr (kVals != kValsNone) mb[moff + 512 * j] = meta_byte;
      if (a.mask_out) ob[m0 * 16 + bb + 512 * j] = static_cast<uint8_t>(keep);
    }
    __syncthreads();   // stage `st` fully read; chunk buffers complete
    if (tid == 0 && i + kStreamStages < nmine) {
      fence_async_shared();
      issue(i + kStreamStages);
    }
    if constexpr (kVals != kValsNone) {
      if (tid < 128) {
        uint4* dst = reinterpret_cast<uint4*>(
            a.meta + (static_cast<int64_t>(rt) * a.kblocks + kb) * 2048);
        __stcs(dst + tid, reinterpret_cast<const uint4*>(mb)[tid]);
      }
    }
    // mask rows of the chunk: threads 256..383 the (second-stage) mask,
    // threads 384..511 the first-stage mask of the progressive kernel
    uint8_t* const mdst = tid < 384 ? a.mask_out : a.mask1_out;
    const uint8_t* const msrc = tid < 384 ? ob : ob1;
    if (mdst && tid >= 256 && (kProg || tid < 384)) {
      const int m = (tid - 256) & 127;
      const int64_t row = static_cast<int64_t>(rt) * 128 + m;
      const int64_t v0 = static_cast<int64_t>(kb) * 16;
      int nb = static_cast<int>(kvec - v0 < 16 ? kvec - v0 : 16);
      if (row < a.n && nb > 0) {
        uint8_t* dst = mdst + row * kvec + v0;
        if (nb == 16 && (reinterpret_cast<uintptr_t>(dst) & 15u) == 0) {
          *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(msrc + m * 16);
        } else {
          for (int e = 0; e < nb; ++e) dst[e] = msrc[m * 16 + e];
        }
      }
    }
  }
  if (bad) raise_error(kErrPatternBit);
}

// --------------------------------------------------------- a5 weight scale
// One warp per row (8 rows per 256-thread block).  Keys = |w| bit patterns (15
// bits) of the kept positions.  One pass gives the kept count c and the
// largest key; when the nearest rank r = ceil(coverage * c) equals c that is
// the answer.  Otherwise the r-th smallest key is found exactly with two
// histogram passes in the warp's shared-memory histogram (high 8 bits, then
// low 7 bits inside the selected bucket) and warp-parallel prefix scans.

// First bin b (of nb, lanes hold nb/32 consecutive bins each) whose inclusive
// prefix count reaches `rank`; returns b and the count below it.
__device__ __forceinline__ uint32_t warp_find_bin(const uint32_t* h, uint32_t nb, uint32_t rank,
                                                  uint32_t& below) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t per = nb / 32u;
  uint32_t local = 0;
  for (uint32_t i = 0; i < per; ++i) local += h[lane * per + i];
  uint32_t incl = local;   // inclusive warp scan of the lane totals
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= static_cast<uint32_t>(o)) incl += t;
  }
  const uint32_t excl = incl - local;
  const uint32_t hit = __ballot_sync(0xFFFFFFFFu, incl >= rank && excl < rank);
  const uint32_t src = __ffs(hit) - 1u;
  uint32_t b = 0, acc = __shfl_sync(0xFFFFFFFFu, excl, src);
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t cnt = h[src * per + i];
    if (acc + cnt >= rank) { b = src * per + i; break; }
    acc += cnt;
  }
  below = acc;
  return b;
}

__global__ void __launch_bounds__(256) wscale_kernel(const uint16_t* __restrict__ w,
                                                     const uint8_t* __restrict__ mask, int64_t n,
                                                     int64_t k, double coverage,
                                                     float* __restrict__ s_w) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ uint32_t hist[8][256];
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t wid = threadIdx.x >> 5;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + wid;
  if (row >= n) return;                                  // whole warp leaves together
  const uint16_t* wr = w + row * k;
  const uint8_t* mr = mask + row * (k / 8);
  const int64_t kvec = k / 8;
  uint32_t* h = hist[wid];

  uint32_t cnt = 0, kmax = 0;
#pragma unroll 4
  for (int64_t v = lane; v < kvec; v += 32) {
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(wr) + v);
    const uint32_t keep = mr[v];
    const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((keep >> i) & 1u) {
        const uint32_t key = mag_key((i & 1) ? (words[i / 2] >> 16) : words[i / 2]);
        kmax = max(kmax, key);
        ++cnt;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    cnt += __shfl_xor_sync(0xFFFFFFFFu, cnt, o);
    kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
  }
  uint32_t key = 0;
  if (cnt > 0) {
    double rd = ceil(coverage * static_cast<double>(cnt));
    uint32_t r = rd < 1.0 ? 1u : static_cast<uint32_t>(rd);
    if (r > cnt) r = cnt;
    if (r == cnt) {
      key = kmax;
    } else {
      for (uint32_t i = lane; i < 256; i += 32) h[i] = 0;
      __syncwarp();
      for (int64_t v = lane; v < kvec; v += 32) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(wr) + v);
        const uint32_t keep = mr[v];
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if ((keep >> i) & 1u)
            atomicAdd(&h[mag_key((i & 1) ? (words[i / 2] >> 16) : words[i / 2]) >> 7], 1u);
      }
      __syncwarp();
      uint32_t below = 0;
      const uint32_t bucket = warp_find_bin(h, 256, r, below);
      const uint32_t r2 = r - below;
      __syncwarp();
      for (uint32_t i = lane; i < 256; i += 32) h[i] = 0;
      __syncwarp();
      for (int64_t v = lane; v < kvec; v += 32) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(wr) + v);
        const uint32_t keep = mr[v];
        const uint32_t words[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((keep >> i) & 1u) {
            const uint32_t kk = mag_key((i & 1) ? (words[i / 2] >> 16) : words[i / 2]);
            if ((kk >> 7) == bucket) atomicAdd(&h[kk & 0x7Fu], 1u);
          }
        }
      }
      __syncwarp();
      uint32_t below2 = 0;
      key = (bucket << 7) | warp_find_bin(h, 128, r2, below2);
    }
  }
  if (lane == 0) {
    const float t = __uint_as_float(key << 16);
    s_w[row] = (cnt == 0 || t == 0.0f) ? 1.0f : __fdiv_rn(t, 127.0f);
  }
}

// ----------------------------------------------------- a5 activation scale
// Exact selection of the r-th smallest |x| over a float32 tensor, on keys =
// bits & 0x7FFFFFFF (monotone in |x| for finite x).
//
// Fast path (large tensors), exact whenever it reports success:
//  1. act_sample_load / act_sample_select: a histogram of kActSample keys at
//     stratified, hashed positions; the histogram bins around the sample rank
//     of r (six standard deviations of a binomial count on each side) give
//     the bracket [lo, hi].
//  2. act_bracket: one pass over the tensor counts keys < lo and appends the
//     keys in [lo, hi] to a candidate list.
//  3. act_bracket_select: if  below < r <= below + candidates  (and the list
//     did not overflow) the answer is the (r - below)-th smallest candidate,
//     selected exactly; otherwise nothing is decided.
// Fallback (small tensors, or a bracket that missed): three radix passes of
// 11/11/9 bits over the whole tensor; every fallback kernel returns at once
// when the fast path already decided.
constexpr int kActSample = 16384;
constexpr uint32_t kActCandCap = 1u << 20;
constexpr int64_t kActBracketMin = int64_t(1) << 18;   // smaller tensors: radix only

struct ActScaleWs {
  uint32_t hist[2048];   // radix histogram
  uint32_t prefix;       // radix: selected high bits so far
  uint32_t rank;         // radix: remaining 1-based rank within the prefix
  uint32_t lo, hi;       // bracket keys (inclusive)
  uint32_t below;        // keys < lo
  uint32_t ncand;        // keys in [lo, hi] (counts past the capacity)
  uint32_t done;         // 1 once s_x holds the answer
  uint32_t blocks_done;  // radix pass: CTAs finished (the last one selects)
  uint32_t fine[4096];   // bracket pass: candidates per fine bin (see act_fine_bin)
  uint32_t cand[kActCandCap];
};

// Fine bin of a candidate key >= lo: 2048 bins per binary exponent over the
// two exponents starting at lo's (the top 11 mantissa bits), keys beyond in
// the last bin.  base = lo with its mantissa cleared.  Every key of a bin
// b < 4095 agrees with base + (b << 12) on bits 12 and up.
constexpr uint32_t kActFineBins = 4096;
__device__ __forceinline__ uint32_t act_fine_bin(uint32_t key, uint32_t base) {
  const uint32_t b = (key - base) >> 12;
  return b < kActFineBins - 1 ? b : kActFineBins - 1;
}

// Inclusive prefix sum of v over a block of 1024 threads (scratch: 32 words).
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = scratch[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    scratch[lane] = w;
  }
  __syncthreads();
  if (warp > 0) v += scratch[warp - 1];
  __syncthreads();
  return v;
}

// k-th smallest (1-based; 1 <= k <= n) of the n keys key_at(0 .. n-1), by a
// block of 1024 threads: radix passes of up to 11 bits over a shared
// histogram, from bit top-1 down to bit 0.  All keys must agree with `fixed`
// on the bits at and above `top` (for unconstrained 31-bit keys: top = 31,
// fixed = 0).  hist: 2048 words; scratch: 34 words.
template <class KeyAt>
__device__ uint32_t block_select(KeyAt key_at, uint32_t n, uint32_t k, uint32_t* hist,
                                 uint32_t* scratch, int top = 31, uint32_t fixed = 0) {
  uint32_t prefix = top >= 31 ? 0u : (fixed & ~((1u << top) - 1u));
  uint32_t mask = top >= 31 ? 0u : (0x7FFFFFFFu & ~((1u << top) - 1u));
  while (top > 0) {
    const int shift = top > 11 ? top - 11 : 0;
    const uint32_t nb = 1u << (top - shift);
    for (uint32_t i = threadIdx.x; i < 2048; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < n; i += blockDim.x) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1u)], 1u);
    }
    __syncthreads();
    const uint32_t b0 = 2u * threadIdx.x;
    const uint32_t h0 = b0 < nb ? hist[b0] : 0u;
    const uint32_t h1 = b0 + 1u < nb ? hist[b0 + 1u] : 0u;
    const uint32_t incl = block_incl_scan(h0 + h1, scratch);
    const uint32_t excl = incl - h0 - h1;
    if (excl < k && k <= incl) {   // exactly one thread holds the k-th key's bin
      const bool second = k > excl + h0;
      scratch[32] = b0 + (second ? 1u : 0u);
      scratch[33] = excl + (second ? h0 : 0u);
    }
    __syncthreads();
    const uint32_t bin = scratch[32], below = scratch[33];
    __syncthreads();
    prefix |= bin << shift;
    mask |= (nb - 1u) << shift;
    k -= below;
    top = shift;
  }
  return prefix;
}

__device__ __forceinline__ uint32_t abs_key(float v) { return __float_as_uint(v) & 0x7FFFFFFFu; }

__device__ __forceinline__ uint32_t mix32(uint32_t v) {   // integer hash (xorshift-multiply)
  v ^= v >> 16;
  v *= 0x7feb352du;
  v ^= v >> 15;
  v *= 0x846ca68bu;
  v ^= v >> 16;
  return v;
}

__global__ void act_scale_init(ActScaleWs* ws, uint32_t rank) {
  pdl_launch_dependents();
  pdl_wait_prior();
  for (int i = threadIdx.x; i < 2048; i += blockDim.x) ws->hist[i] = 0;
  if (threadIdx.x == 0) {
    ws->prefix = 0;
    ws->rank = rank;
    ws->done = 0;
    ws->blocks_done = 0;
  }
}

// Sample: kActSample keys at stratified, hashed positions (stratum i =
// [i * stride, (i + 1) * stride), stride = count / kActSample in [16, 2^17],
// offset = a hash of i scaled to the stratum), one per thread of
// kActSampleCtas CTAs so that the scattered loads spread over many SMs.  Each
// CTA writes the histogram of its keys' top 11 bits (bits 30..20: exponent
// and 3 mantissa bits) to its own 2048-word slice at the start of the
// candidate list (which act_bracket overwrites afterwards).
constexpr int kActSampleCtas = kActSample / 1024;

__global__ void __launch_bounds__(1024) act_sample_load(const float* __restrict__ x,
                                                        int64_t count, ActScaleWs* ws) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ uint32_t h[2048];
  h[threadIdx.x] = 0;
  h[threadIdx.x + 1024] = 0;
  __syncthreads();
  const uint32_t stride = static_cast<uint32_t>(count / kActSample);
  const uint32_t i = blockIdx.x * 1024u + threadIdx.x;
  const uint32_t off = __umulhi(mix32(i), stride);
  const uint32_t key = abs_key(__ldg(x + (static_cast<int64_t>(i) * stride + off)));
  atomicAdd(&h[key >> 20], 1u);
  __syncthreads();
  uint32_t* out = ws->cand + blockIdx.x * 2048u;
  out[threadIdx.x] = h[threadIdx.x];
  out[threadIdx.x + 1024] = h[threadIdx.x + 1024];
}

// Sums the per-CTA sample histograms and brackets the target: lo = lower edge
// of the bin holding sample rank rs - half, hi = upper edge of the bin holding
// rs + half (six binomial standard deviations of the sample count on each
// side; 0 / all-ones when the rank falls off the sample).  The bracket only
// has to be likely: act_bracket_select checks it exactly.
__global__ void __launch_bounds__(1024) act_sample_select(int64_t count, uint32_t rank,
                                                          ActScaleWs* ws) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ uint32_t scratch[34];
  __shared__ uint32_t bins[2];
  const uint32_t b0 = 2u * threadIdx.x;
  uint32_t h0 = 0, h1 = 0;
#pragma unroll
  for (int c = 0; c < kActSampleCtas; ++c) {
    h0 += __ldcg(ws->cand + c * 2048 + b0);
    h1 += __ldcg(ws->cand + c * 2048 + b0 + 1);
  }
  for (int i = threadIdx.x; i < 2048; i += blockDim.x) ws->hist[i] = 0;
  const double q = static_cast<double>(rank) / static_cast<double>(count);
  const double sd = sqrt(static_cast<double>(kActSample) * q * (1.0 - q));
  const int64_t half = static_cast<int64_t>(ceil(6.0 * sd)) + 4;
  int64_t rs = static_cast<int64_t>(ceil(q * kActSample));
  rs = rs < 1 ? 1 : (rs > kActSample ? kActSample : rs);
  const bool has_lo = rs - half >= 1, has_hi = rs + half <= kActSample;
  const uint32_t k_lo = has_lo ? static_cast<uint32_t>(rs - half) : 1u;
  const uint32_t k_hi = has_hi ? static_cast<uint32_t>(rs + half) : 1u;
  const uint32_t incl = block_incl_scan(h0 + h1, scratch);
  const uint32_t excl = incl - h0 - h1;
  if (excl < k_lo && k_lo <= incl) bins[0] = b0 + (k_lo > excl + h0 ? 1u : 0u);
  if (excl < k_hi && k_hi <= incl) bins[1] = b0 + (k_hi > excl + h0 ? 1u : 0u);
  __syncthreads();
  for (int i = threadIdx.x; i < static_cast<int>(kActFineBins); i += blockDim.x) ws->fine[i] = 0;
  if (threadIdx.x == 0) {
    ws->lo = has_lo ? bins[0] << 20 : 0u;
    ws->hi = has_hi ? (bins[1] << 20) | 0xFFFFFu : 0xFFFFFFFFu;
    ws->below = 0;
    ws->ncand = 0;
    ws->done = 0;
    ws->prefix = 0;
    ws->rank = rank;
    ws->blocks_done = 0;
  }
}

constexpr int kActLocalCap = 2048;   // candidates one CTA buffers in shared memory

__device__ __forceinline__ void bracket_one(uint32_t key, uint32_t lo, uint32_t hi,
                                            uint32_t& below, uint32_t* buf, uint32_t* nbuf) {
  below += key < lo ? 1u : 0u;
  if (key >= lo && key <= hi) {   // rare: a few candidates per CTA
    const uint32_t i = atomicAdd(nbuf, 1u);
    if (i < kActLocalCap) buf[i] = key;
  }
}

// One pass: keys < lo are counted, keys in [lo, hi] are collected per CTA in
// shared memory and appended to the workspace list with one reservation per
// CTA.  A CTA that finds more than kActLocalCap candidates makes the list
// count exceed its capacity, which sends the decision to the radix fallback.
__global__ void __launch_bounds__(256) act_bracket(const float4* __restrict__ x, int64_t nvec,
                                                   const float* __restrict__ tail, int ntail,
                                                   ActScaleWs* ws) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ uint32_t buf[kActLocalCap];
  __shared__ uint32_t nbuf, base, part[8];
  if (threadIdx.x == 0) nbuf = 0;
  __syncthreads();
  const uint32_t lo = ws->lo, hi = ws->hi;
  uint32_t below = 0;
  constexpr int kU = 8;   // float4 loads in flight per thread
  const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; v + (kU - 1) * step < nvec; v += kU * step) {
    float4 q[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) q[u] = __ldcs(x + v + u * step);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      bracket_one(abs_key(q[u].x), lo, hi, below, buf, &nbuf);
      bracket_one(abs_key(q[u].y), lo, hi, below, buf, &nbuf);
      bracket_one(abs_key(q[u].z), lo, hi, below, buf, &nbuf);
      bracket_one(abs_key(q[u].w), lo, hi, below, buf, &nbuf);
    }
  }
  for (; v < nvec; v += step) {
    const float4 q = __ldcs(x + v);
    bracket_one(abs_key(q.x), lo, hi, below, buf, &nbuf);
    bracket_one(abs_key(q.y), lo, hi, below, buf, &nbuf);
    bracket_one(abs_key(q.z), lo, hi, below, buf, &nbuf);
    bracket_one(abs_key(q.w), lo, hi, below, buf, &nbuf);
  }
  if (blockIdx.x == 0 && static_cast<int>(threadIdx.x) < ntail)
    bracket_one(abs_key(tail[threadIdx.x]), lo, hi, below, buf, &nbuf);
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
  if (lane == 0) part[threadIdx.x >> 5] = below;
  __syncthreads();
  const uint32_t n = nbuf;
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int w = 0; w < (blockDim.x >> 5); ++w) t += part[w];
    if (t) atomicAdd(&ws->below, t);
    // an overflowing CTA pushes the count past the capacity (fallback decides)
    base = n == 0 ? 0u : atomicAdd(&ws->ncand, n <= kActLocalCap ? n : kActCandCap + 1u);
  }
  __syncthreads();
  if (n <= kActLocalCap)
    for (uint32_t i = threadIdx.x; i < n; i += blockDim.x)
      if (base + i < kActCandCap) ws->cand[base + i] = buf[i];
  // each candidate also counts in its fine bin (for the final selection)
  if (n <= kActLocalCap) {
    const uint32_t fbase = lo & 0x7F800000u;
    for (uint32_t i = threadIdx.x; i < n; i += blockDim.x)
      atomicAdd(&ws->fine[act_fine_bin(buf[i], fbase)], 1u);
  }
}

// Candidates staged in dynamic shared memory when they fit (kActSelSmemKeys),
// else read from the workspace list in every radix pass.
constexpr uint32_t kActSelSmemKeys = 48 * 1024;

__global__ void __launch_bounds__(1024) act_bracket_select(ActScaleWs* ws, float* s_x) {
  pdl_launch_dependents();
  pdl_wait_prior();
  extern __shared__ uint32_t ck[];
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t scratch[34];
  const uint32_t below = ws->below, n = ws->ncand, rank = ws->rank;
  if (!(below < rank && rank - below <= n && n <= kActCandCap)) return;   // radix decides
  const uint32_t* cand = ws->cand;
  // fine bin holding the (rank - below)-th candidate, from the bracket pass's
  // histogram: 4 bins per thread, one block scan
  {
    const uint32_t k = rank - below;
    uint32_t h[4], local = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      h[j] = __ldcg(ws->fine + 4 * threadIdx.x + j);
      local += h[j];
    }
    const uint32_t incl = block_incl_scan(local, scratch);
    uint32_t acc = incl - local;
    if (acc < k && k <= incl) {
      uint32_t b = 4 * threadIdx.x;
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        if (acc + h[j] >= k) break;
        acc += h[j];
        ++b;
      }
      scratch[32] = b;
      scratch[33] = acc;
      scratch[31] = h[b - 4 * threadIdx.x];
    }
    __syncthreads();
    const uint32_t bin = scratch[32], before = scratch[33], cnt = scratch[31];
    __syncthreads();
    // every key of a bin below the last agrees on bits 12 and up: select
    // among that bin's candidates only
    if (bin < kActFineBins - 1 && cnt <= kActSelSmemKeys) {
      const uint32_t fbase = ws->lo & 0x7F800000u;
      __shared__ uint32_t nsel;
      if (threadIdx.x == 0) nsel = 0;
      __syncthreads();
      // eight loads in flight per thread, then the (rare) appends
      constexpr int kU = 8;
      for (uint32_t i0 = threadIdx.x; i0 < n; i0 += kU * blockDim.x) {
        uint32_t v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const uint32_t i = i0 + u * blockDim.x;
          v[u] = i < n ? __ldcg(cand + i) : 0xFFFFFFFFu;
        }
#pragma unroll
        for (int u = 0; u < kU; ++u)
          if (v[u] != 0xFFFFFFFFu && act_fine_bin(v[u], fbase) == bin)
            ck[atomicAdd(&nsel, 1u)] = v[u];
      }
      __syncthreads();
      const uint32_t fixed = fbase + (bin << 12);
      const uint32_t key = block_select([&](uint32_t j) { return ck[j]; }, cnt, k - before, hist,
                                        scratch, 12, fixed);
      if (threadIdx.x == 0) {
        const float t = __uint_as_float(key);
        *s_x = (t == 0.0f) ? 1.0f : __fdiv_rn(t, 127.0f);
        ws->done = 1;
      }
      return;
    }
  }
  // every candidate lies in [lo, max]: only the bits below the highest bit in
  // which lo and the largest candidate differ can vary
  __shared__ uint32_t wmax[32];
  uint32_t key;
  if (n <= kActSelSmemKeys) {
    constexpr int kU = 8;
    uint32_t kmax = 0;
    uint32_t i = threadIdx.x;
    for (; i + (kU - 1) * 1024 < n; i += kU * 1024) {
      uint32_t v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) v[u] = cand[i + u * 1024];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        ck[i + u * 1024] = v[u];
        kmax = v[u] > kmax ? v[u] : kmax;
      }
    }
    for (; i < n; i += 1024) {
      const uint32_t v = cand[i];
      ck[i] = v;
      kmax = v > kmax ? v : kmax;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = kmax;
    __syncthreads();
    kmax = wmax[threadIdx.x & 31];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    const uint32_t diff = (ws->lo ^ kmax) & 0x7FFFFFFFu;
    const int top = diff ? 32 - __clz(diff) : 0;
    key = block_select([&](uint32_t j) { return ck[j]; }, n, rank - below, hist, scratch, top,
                       ws->lo);
  } else {
    const uint32_t diff = (ws->lo ^ ws->hi) & 0x7FFFFFFFu;
    const int top = diff ? 32 - __clz(diff) : 0;
    key = block_select([&](uint32_t j) { return cand[j]; }, n, rank - below, hist, scratch, top,
                       ws->lo);
  }
  if (threadIdx.x == 0) {
    const float t = __uint_as_float(key);
    *s_x = (t == 0.0f) ? 1.0f : __fdiv_rn(t, 127.0f);
    ws->done = 1;
  }
}

// Radix pass p of the fallback: per-CTA shared histograms of bits [shift,
// shift + bits) of the keys under the current prefix, merged into the
// workspace; the last CTA to finish picks the bin holding the rank, narrows
// the prefix and clears the histogram for the next pass (writing s_x after
// the last pass).  Returns at once when the bracket path has decided.
__global__ void __launch_bounds__(256) act_scale_hist(const float4* __restrict__ x, int64_t nvec,
                                                      const float* __restrict__ tail,
                                                      int ntail, ActScaleWs* ws, int shift,
                                                      int bits, uint32_t hi_mask, float* s_x,
                                                      int last_pass) {
  pdl_launch_dependents();
  pdl_wait_prior();
  if (ws->done) return;
  __shared__ uint32_t h[2048];
  __shared__ uint32_t is_last;
  const uint32_t nb = 1u << bits;
  for (uint32_t i = threadIdx.x; i < nb; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const uint32_t prefix = ws->prefix;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec;
       v += stride) {
    const float4 q = __ldcs(x + v);
    const float e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t key = abs_key(e[i]);
      if ((key & hi_mask) == prefix) atomicAdd(&h[(key >> shift) & (nb - 1u)], 1u);
    }
  }
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < ntail; i += blockDim.x) {
      const uint32_t key = abs_key(tail[i]);
      if ((key & hi_mask) == prefix) atomicAdd(&h[(key >> shift) & (nb - 1u)], 1u);
    }
  }
  __syncthreads();
  for (uint32_t i = threadIdx.x; i < nb; i += blockDim.x)
    if (h[i]) atomicAdd(&ws->hist[i], h[i]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = atomicAdd(&ws->blocks_done, 1u) == gridDim.x - 1u;
  __syncthreads();
  if (!is_last || threadIdx.x != 0) return;
  __threadfence();
  volatile uint32_t* vh = ws->hist;
  uint32_t below = 0, b = 0;
  for (b = 0; b < nb - 1u; ++b) {
    if (below + vh[b] >= ws->rank) break;
    below += vh[b];
  }
  ws->prefix |= b << shift;
  ws->rank -= below;
  for (uint32_t i = 0; i < nb; ++i) vh[i] = 0;
  ws->blocks_done = 0;
  if (last_pass) {
    const float t = __uint_as_float(ws->prefix);
    *s_x = (t == 0.0f) ? 1.0f : __fdiv_rn(t, 127.0f);
  }
}

// ----------------------------------------------------------- quantisation
// q = clamp(rint(x / s), -127, 127) with x / s the correctly rounded float32
// quotient.  y = x * rcp(s) is within a few ulps of that quotient, so rint(y)
// equals rint(x / s) unless a half-integer lies within that distance of y;
// there (and for non-finite y) the quotient is formed exactly.
__device__ __forceinline__ uint32_t q8(float x, float s, float rs) {
  const float y = __fmul_rn(x, rs);
  const float f = y - floorf(y);
  float d = y;
  if (!(fabsf(f - 0.5f) > 1e-5f * fabsf(y) + 1e-30f)) d = __fdiv_rn(x, s);
  int q = __float2int_rn(d);
  q = q > 127 ? 127 : (q < -127 ? -127 : q);
  return static_cast<uint32_t>(q) & 0xFFu;
}

__global__ void __launch_bounds__(256) quantize_kernel(const float4* __restrict__ x, int64_t nvec16,
                                                       const float* __restrict__ s_ptr,
                                                       uint4* __restrict__ xq) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const float s = *s_ptr;
  const float rs = __frcp_rn(s);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < nvec16;
       v += stride) {
    float4 in[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) in[j] = __ldcs(x + 4 * v + j);
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float4 q = in[j];
      out[j] = q8(q.x, s, rs) | (q8(q.y, s, rs) << 8) | (q8(q.z, s, rs) << 16) |
               (q8(q.w, s, rs) << 24);
    }
    xq[v] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__global__ void quantize_tail(const float* __restrict__ x, int64_t start, int64_t count,
                              const float* __restrict__ s_ptr, int8_t* __restrict__ xq) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const int64_t i = start + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < count) xq[i] = static_cast<int8_t>(q8(x[i], *s_ptr, __frcp_rn(*s_ptr)));
}


// ------------------------------------------- Sparse-QAT fake quantisation
// [Ampere-sparsity] "PTQ and QAT": the forward pass of quantisation-aware
// training quantises the weights to int8 and dequantises them back.  For the
// masked weights: kept -> bf16(float(q) * s_w[row]) with q the int8 code of
// the inference quantiser (q8), dropped -> +0.  One thread per 8 weights of a
// row (16-byte load and store; bit j of the mask byte is weight j).
__device__ __forceinline__ uint32_t fake_quant_one(uint32_t bits16, bool kept, float s, float rs) {
  if (!kept) return 0u;
  const int q = static_cast<int8_t>(q8(__uint_as_float(bits16 << 16), s, rs) & 0xFFu);
  const float f = __fmul_rn(__int2float_rn(q), s);
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(f)));
}

__global__ void __launch_bounds__(256) fake_quant_kernel(const uint4* __restrict__ w,
                                                         const uint8_t* __restrict__ mask,
                                                         const float* __restrict__ s_w, int64_t n,
                                                         int64_t kvec, uint4* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait_prior();
  for (int64_t row = blockIdx.y; row < n; row += gridDim.y) {
    const float s = __ldg(s_w + row);
    const float rs = __frcp_rn(s);
    for (int64_t v = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; v < kvec;
         v += static_cast<int64_t>(gridDim.x) * blockDim.x) {
      const int64_t i = row * kvec + v;
      const uint4 q = __ldcs(w + i);
      const uint32_t m = __ldg(mask + i);
      const uint32_t words[4] = {q.x, q.y, q.z, q.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t lo = fake_quant_one(words[e] & 0xFFFFu, (m >> (2 * e)) & 1u, s, rs);
        const uint32_t hi = fake_quant_one(words[e] >> 16, (m >> (2 * e + 1)) & 1u, s, rs);
        o[e] = lo | (hi << 16);
      }
      __stcs(out + i, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// ------------------------------------ a2..a5 INT8 weight conversion, one pass
// Magnitude 2:4 pruning, the per-row weight scale and the int8 compression of
// W in one kernel: the outputs of sp24_prune (n_keep = 2), sp24_wscale and
// sp24_compress(SP24_INT8) without their three passes over W.  One warp per
// row (8 rows per 256-thread block):
//  * pass 1 reads the row and takes its largest |w| key.  The largest
//    magnitude of a group is always kept, so this is the largest kept key;
//    every group keeps exactly two positions, so the kept count c = K/2 and
//    the nearest rank r = max(1, ceil(coverage * c)) are known up front.  When
//    r = c the scale is that maximum; otherwise the weight-scale kernel's two
//    histogram passes over the kept keys select the r-th smallest;
//  * pass 2 reads the row again (its bytes are still in L2) and writes the
//    keep mask, the int8 values (q8, the quantiser of sp24_compress) and the
//    metadata bytes.  Positions >= K up to the 128-position chunk and rows
//    >= N up to the 128-row tile get the padding pattern (0, 1), as
//    sp24_compress writes them.
template <class F>
__device__ __forceinline__ void for_kept_keys(const uint4* wr, int64_t kvec, uint32_t lane, F&& f) {
  for (int64_t v = lane; v < kvec; v += 32) {
    const uint4 q = __ldg(wr + v);
    uint32_t lo0, hi0, lo1, hi1;
    top2_positions_mag<false>(q.x, q.y, 0xFu, lo0, hi0);
    top2_positions_mag<false>(q.z, q.w, 0xFu, lo1, hi1);
    const uint32_t p0 = gather_pair(q.x, q.y, lo0, hi0);
    const uint32_t p1 = gather_pair(q.z, q.w, lo1, hi1);
    f(mag_key(p0));
    f(mag_key(p0 >> 16));
    f(mag_key(p1));
    f(mag_key(p1 >> 16));
  }
}

// Writes the outputs of one row's vector v (8 weights) given the row scale.
__device__ __forceinline__ void int8_emit(const uint4& q, int64_t v, float s, float rs,
                                          uint32_t* vr, uint8_t* mr, uint8_t* mrow) {
  uint32_t lo0, hi0, lo1, hi1;
  top2_positions_mag<false>(q.x, q.y, 0xFu, lo0, hi0);
  top2_positions_mag<false>(q.z, q.w, 0xFu, lo1, hi1);
  const uint32_t p0 = gather_pair(q.x, q.y, lo0, hi0);
  const uint32_t p1 = gather_pair(q.z, q.w, lo1, hi1);
  const uint32_t packed = q8(__uint_as_float(p0 << 16), s, rs) |
                          (q8(__uint_as_float(p0 & 0xFFFF0000u), s, rs) << 8) |
                          (q8(__uint_as_float(p1 << 16), s, rs) << 16) |
                          (q8(__uint_as_float(p1 & 0xFFFF0000u), s, rs) << 24);
  __stcs(vr + v, packed);
  if (mr) mr[v] = static_cast<uint8_t>((1u << lo0) | (1u << hi0) | (((1u << lo1) | (1u << hi1)) << 4));
  mrow[(v >> 4) * 2048 + (v & 15)] = static_cast<uint8_t>(lo0 | (hi0 << 2) | (lo1 << 4) | (hi1 << 6));
}

__device__ __forceinline__ uint32_t vec_max_key(const uint4& q) {
  const uint32_t m0 = max(mag_key(q.x), mag_key(q.x >> 16));
  const uint32_t m1 = max(mag_key(q.y), mag_key(q.y >> 16));
  const uint32_t m2 = max(mag_key(q.z), mag_key(q.z >> 16));
  const uint32_t m3 = max(mag_key(q.w), mag_key(q.w >> 16));
  return max(max(m0, m1), max(m2, m3));
}

// The r-th smallest kept key of a row (r < kept count): two histogram passes
// over the kept keys, as the weight-scale kernel.
__device__ __forceinline__ uint32_t int8_select_key(const uint4* wr, int64_t kvec, uint32_t r,
                                                    uint32_t* h, uint32_t lane) {
  for (uint32_t i = lane; i < 256; i += 32) h[i] = 0;
  __syncwarp();
  for_kept_keys(wr, kvec, lane, [&](uint32_t kk) { atomicAdd(&h[kk >> 7], 1u); });
  __syncwarp();
  uint32_t below = 0;
  const uint32_t bucket = warp_find_bin(h, 256, r, below);
  const uint32_t r2 = r - below;
  __syncwarp();
  for (uint32_t i = lane; i < 256; i += 32) h[i] = 0;
  __syncwarp();
  for_kept_keys(wr, kvec, lane, [&](uint32_t kk) {
    if ((kk >> 7) == bucket) atomicAdd(&h[kk & 0x7Fu], 1u);
  });
  __syncwarp();
  uint32_t below2 = 0;
  return (bucket << 7) | warp_find_bin(h, 128, r2, below2);
}

// Two warps per row (4 rows per 256-thread block), each taking every other
// group of 32 vectors of the row: half h handles vectors lane + 32 * (2 i + h).
// kHalfVec > 0: a half (at most 32 * kHalfVec vectors) stays in registers
// between the passes, all its loads in flight at once; 0: any K, the half is
// read in batches of 8 vectors per lane and again for the output pass.
constexpr int kInt8HalfVec = 8;   // rows up to K = 4096 in registers

template <int kHalfVec>
__global__ void __launch_bounds__(256) prune_int8_kernel(const uint16_t* __restrict__ w, int64_t n,
                                                         int64_t k, double coverage,
                                                         uint8_t* __restrict__ mask_out,
                                                         float* __restrict__ s_w,
                                                         uint32_t* __restrict__ vals,
                                                         uint8_t* __restrict__ meta) {
  pdl_launch_dependents();
  pdl_wait_prior();
  __shared__ uint32_t hist[4][256];
  __shared__ uint32_t half_max[8];
  __shared__ uint32_t row_key[4];
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t wid = threadIdx.x >> 5;
  const uint32_t slot = wid >> 1;        // row within the block
  const uint32_t half = wid & 1u;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + slot;
  const bool live = row < n;             // rows >= n: padding of the last 128-row tile
  const int64_t kvec = k / 8;
  const int kblocks = static_cast<int>((k + 127) / 128);
  const int64_t kvec_pad = static_cast<int64_t>(kblocks) * 16;
  // metadata of this row: chunk kb at + kb * 2048, vector bb of the chunk at + bb
  uint8_t* mrow = meta + (row >> 7) * kblocks * 2048 + 16 * (row & 127);
  const uint4* wr = reinterpret_cast<const uint4*>(w + (live ? row : 0) * k);
  // vector of this lane's i-th slot
  auto vec_of = [&](int64_t i) { return static_cast<int64_t>(lane) + 32 * (2 * i + half); };
  const int64_t nslots = (kvec + 63) / 64;   // slots per lane over the row

  uint4 reg[kHalfVec > 0 ? kHalfVec : 1];
  uint32_t kmax = 0;
  if (live) {
    if constexpr (kHalfVec > 0) {
#pragma unroll
      for (int i = 0; i < kHalfVec; ++i) {
        const int64_t v = vec_of(i);
        reg[i] = v < kvec ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int i = 0; i < kHalfVec; ++i) kmax = max(kmax, vec_max_key(reg[i]));
    } else {
      for (int64_t i0 = 0; i0 < nslots; i0 += 8) {
        uint4 b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t v = vec_of(i0 + i);
          b[i] = v < kvec ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) kmax = max(kmax, vec_max_key(b[i]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xFFFFFFFFu, kmax, o));
    if (lane == 0) half_max[wid] = kmax;
  }
  __syncthreads();
  const uint32_t cnt = static_cast<uint32_t>(kvec * 4);
  uint32_t r = cnt;
  {
    const double rd = ceil(coverage * static_cast<double>(cnt));
    r = rd < 1.0 ? 1u : static_cast<uint32_t>(rd);
    if (r > cnt) r = cnt;
  }
  // the r-th smallest kept key: the row maximum when r = c, else selected by
  // the row's first warp over the whole row
  if (live && half == 0) {
    uint32_t key = max(half_max[2 * slot], half_max[2 * slot + 1]);
    if (r < cnt) key = int8_select_key(wr, kvec, r, hist[slot], lane);
    if (lane == 0) row_key[slot] = key;
  }
  __syncthreads();
  if (live) {
    const uint32_t key = row_key[slot];
    const float t = __uint_as_float(key << 16);
    const float s = (cnt == 0 || t == 0.0f) ? 1.0f : __fdiv_rn(t, 127.0f);
    if (half == 0 && lane == 0) s_w[row] = s;
    const float rs = __frcp_rn(s);
    uint8_t* mr = mask_out ? mask_out + row * kvec : nullptr;
    uint32_t* vr = vals + row * kvec;
    if constexpr (kHalfVec > 0) {
#pragma unroll
      for (int i = 0; i < kHalfVec; ++i) {
        const int64_t v = vec_of(i);
        if (v < kvec) int8_emit(reg[i], v, s, rs, vr, mr, mrow);
      }
    } else {
      for (int64_t i0 = 0; i0 < nslots; i0 += 8) {
        uint4 b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t v = vec_of(i0 + i);
          b[i] = v < kvec ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t v = vec_of(i0 + i);
          if (v < kvec) int8_emit(b[i], v, s, rs, vr, mr, mrow);
        }
      }
    }
  }
  // metadata padding: positions >= K of the last 128-position chunk, and
  // whole rows >= n of the last 128-row tile
  const int64_t pad0 = live ? kvec : 0;
  for (int64_t v = pad0 + lane + 32 * half; v < kvec_pad; v += 64)
    mrow[(v >> 4) * 2048 + (v & 15)] = 0x44u;
}

// ------------------------------------------- Wanda prune without allocation
// For callers that may not allocate device memory (see sp24_prune_wanda_noalloc
// in include/sp24.h): the float64 column norms live in this file-scope array
// instead of a caller workspace.  Every GPU that loads the library holds it
// (SP24_NOALLOC_MAX_K * 8 bytes) until the process exits.
__device__ __align__(256) double g_noalloc_norms[SP24_NOALLOC_MAX_K];

namespace {
constexpr int kNoallocMaxDevices = 64;

// The array's device address on one device, and the context it was looked up
// in.  A module's globals move when its context is destroyed and recreated
// (cudaDeviceReset, for instance), so the address is looked up again whenever
// the device's current context differs from the one recorded here.
struct NoallocSlot {
  CUcontext ctx;
  double* ptr;
};
NoallocSlot g_noalloc_slot[kNoallocMaxDevices];
std::mutex g_noalloc_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

CUcontext current_ctx() {
  CUcontext c = nullptr;
  const CtxGetCurrentFn f = ctx_get_current();
  if (f == nullptr || f(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_norms on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call and after
// any change of the device's context, and cached otherwise.
sp24_status noalloc_norms(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
  if (dev < 0 || dev >= kNoallocMaxDevices) return SP24_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  const CUcontext before = current_ctx();
  if (slot.ptr == nullptr || before == nullptr || before != slot.ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_norms);
    if (e != cudaSuccess) return cuda_fail("cudaGetSymbolAddress", e);
    slot.ptr = static_cast<double*>(p);
    slot.ctx = current_ctx();   // the lookup creates the primary context if needed
  }
  *out = slot.ptr;
  return SP24_OK;
}
}  // namespace

// -------------------------------------------------------------- launching
static int grid_for(int64_t work_items, int threads) {
  const int64_t want = (work_items + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

static sp24_status launch_colnorm(const void* xc, int64_t mc, int64_t k, double* norms,
                                  cudaStream_t s) {
  const int blocks = static_cast<int>((k + 63) / 64);
  return launch_kernel(colnorm_kernel, dim3(blocks), dim3(256), 0, s, 1,
                       static_cast<const uint16_t*>(xc), mc, k, norms);
}

template <bool kPrune, bool kWanda, int kVals, bool kMaskIn, bool kProg = false>
static sp24_status launch_stream_t(const void* w, const uint8_t* mask, uint8_t* mask_out,
                                 const double* norms, const float* s_w, int64_t n, int64_t k,
                                 int n_keep, void* vals, void* meta, cudaStream_t s,
                                 const void* xc, int64_t mc, uint8_t* mask1_out = nullptr) {
  auto kern = stream_kernel<kPrune, kWanda, kVals, kMaskIn, kProg>;
  constexpr int kExtra = kProg ? kProgExtra : 0;
  static std::atomic<uint64_t> smem_set{0};   // one bit per device
  SP24_TRY(set_smem_once(reinterpret_cast<const void*>(kern),
                         (kWanda ? kStreamSmemFused : kStreamSmem) + kExtra, smem_set));
  cudaError_t e = cudaSuccess;
  const int64_t kblocks = (k + 127) / 128;
  const int64_t nchunks = ((n + 127) / 128) * kblocks;
  if (nchunks > 0x7FFFFFFF) return SP24_ERR_UNSUPPORTED;
  CUtensorMap tw, tm, tn, ts;
  SP24_TRY(make_map(&tw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, static_cast<uint64_t>(k),
                    static_cast<uint64_t>(n), 128, 128, CU_TENSOR_MAP_SWIZZLE_NONE));
  // mask bytes ride along with the TMA stage when their rows are 16-byte aligned
  const bool mask_tma = mask != nullptr && (k % 128) == 0;
  tm = tw;
  if (mask_tma)
    SP24_TRY(make_map(&tm, mask, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, static_cast<uint64_t>(k / 8),
                      static_cast<uint64_t>(n), 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE));
  tn = tw;
  if (kWanda && xc == nullptr)
    SP24_TRY(make_map_1d(&tn, norms, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, static_cast<uint64_t>(k),
                         128));
  ts = tw;
  if (kVals == kValsINT8)
    SP24_TRY(make_map_1d(&ts, s_w, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, static_cast<uint64_t>(n),
                         128));
  StreamArgs a;
  a.n = n;
  a.k = k;
  a.kblocks = static_cast<int>(kblocks);
  a.nchunks = static_cast<int>(nchunks);
  a.n_keep = n_keep;
  a.mask_tma = mask_tma ? 1 : 0;
  a.mask_direct = mask_tma ? nullptr : mask;
  a.mask_out = mask_out;
  a.mask1_out = mask1_out;
  a.vals = vals;
  a.meta = static_cast<uint8_t*>(meta);
  a.xc = static_cast<const uint16_t*>(xc);
  a.mc = mc;
  a.norms_out = const_cast<double*>(norms);
  const int smem = ((kWanda && xc != nullptr) ? kStreamSmemFused : kStreamSmem) + kExtra;
  // as many persistent CTAs as fit (two per SM: one's barrier and TMA waits
  // overlap the other's work)
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kStreamThreads, smem);
  if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveBlocksPerMultiprocessor", e);
  if (per_sm < 1) return SP24_ERR_UNSUPPORTED;
  const int64_t ctas = static_cast<int64_t>(sm_count()) * per_sm;
  const int grid = static_cast<int>(nchunks < ctas ? nchunks : ctas);
  return launch_kernel(kern, dim3(grid), dim3(kStreamThreads), smem, s, 1, tw, tm, tn, ts, a);
}

// For the pruning variants `mask` is mask_in (optional); a separate
// instantiation without it drops the liveness selects from the inner loop.
template <bool kPrune, bool kWanda, int kVals>
static sp24_status launch_stream(const void* w, const uint8_t* mask, uint8_t* mask_out,
                                 const double* norms, const float* s_w, int64_t n, int64_t k,
                                 int n_keep, void* vals, void* meta, cudaStream_t s,
                                 const void* xc = nullptr, int64_t mc = 0) {
  if (kPrune && mask == nullptr)
    return launch_stream_t<kPrune, kWanda, kVals, false>(w, mask, mask_out, norms, s_w, n, k,
                                                         n_keep, vals, meta, s, xc, mc);
  return launch_stream_t<kPrune, kWanda, kVals, true>(w, mask, mask_out, norms, s_w, n, k, n_keep,
                                                      vals, meta, s, xc, mc);
}

// Wanda pruning: the column norms go to `norms` either from a separate
// colnorm launch or, when recomputing them per row tile is cheap (row tiles x
// calibration rows small), inside the prune kernel itself (one launch fewer).
constexpr int64_t kFusedNormWork = 8192;   // max row tiles x Mc for the fused path

static sp24_status launch_wanda_prune(const void* W, const uint8_t* mask_in, uint8_t* mask_out,
                                      double* norms, int64_t N, int64_t K, const void* Xc,
                                      int64_t Mc, int n_keep, cudaStream_t s) {
  if (((N + 127) / 128) * Mc <= kFusedNormWork)
    return launch_stream<true, true, kValsNone>(W, mask_in, mask_out, norms, nullptr, N, K, n_keep,
                                                nullptr, nullptr, s, Xc, Mc);
  SP24_TRY(launch_colnorm(Xc, Mc, K, norms, s));
  return launch_stream<true, true, kValsNone>(W, mask_in, mask_out, norms, nullptr, N, K, n_keep,
                                              nullptr, nullptr, s);
}

// Progressive pruning in one pass (3 of 4, then 2 of 4 of the survivors),
// optionally with the bf16 compression of the second mask.  Wanda norms as in
// launch_wanda_prune.
template <int kVals>
static sp24_status launch_progressive(const void* W, int64_t N, int64_t K, const void* Xc,
                                      int64_t Mc, bool wanda, uint8_t* mask1_out,
                                      uint8_t* mask2_out, void* vals, void* meta, double* norms,
                                      cudaStream_t s) {
  if (!wanda)
    return launch_stream_t<true, false, kVals, false, true>(W, nullptr, mask2_out, nullptr,
                                                           nullptr, N, K, 2, vals, meta, s,
                                                           nullptr, 0, mask1_out);
  if (((N + 127) / 128) * Mc <= kFusedNormWork)
    return launch_stream_t<true, true, kVals, false, true>(W, nullptr, mask2_out, norms, nullptr,
                                                          N, K, 2, vals, meta, s, Xc, Mc,
                                                          mask1_out);
  SP24_TRY(launch_colnorm(Xc, Mc, K, norms, s));
  return launch_stream_t<true, true, kVals, false, true>(W, nullptr, mask2_out, norms, nullptr, N,
                                                        K, 2, vals, meta, s, nullptr, 0,
                                                        mask1_out);
}

}  // namespace sp24

using namespace sp24;

extern "C" {

sp24_status sp24_prune_progressive(const void* W, int64_t N, int64_t K, const void* Xc,
                                   int64_t Mc, int mode, uint8_t* mask1_out, uint8_t* mask2_out,
                                   void* vals, void* meta, void* workspace, void* stream) {
  if (N < 0 || K < 0 || (mode != SP24_MAGNITUDE && mode != SP24_WANDA)) return SP24_ERR_ARG;
  if (N == 0 || K == 0) return SP24_OK;
  const bool compress = vals != nullptr || meta != nullptr;
  if (!W || (compress && (!vals || !meta)) || (!compress && !mask1_out && !mask2_out))
    return SP24_ERR_ARG;
  if (mode == SP24_WANDA && (!Xc || Mc < 1 || !workspace)) return SP24_ERR_ARG;
  if (K % (compress ? 16 : 8) != 0) return SP24_ERR_ALIGN;
  if (!aligned16(W) || (mask1_out && !aligned16(mask1_out)) ||
      (mask2_out && !aligned16(mask2_out)) || (vals && !aligned16(vals)) ||
      (meta && !aligned16(meta)))
    return SP24_ERR_ALIGN;
  if (mode == SP24_WANDA && (!aligned16(Xc) || !aligned16(workspace))) return SP24_ERR_ALIGN;
  if ((N + 127) / 128 > 65535) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  double* norms = static_cast<double*>(workspace);
  const bool wanda = mode == SP24_WANDA;
  if (compress)
    return launch_progressive<kValsBF16>(W, N, K, Xc, Mc, wanda, mask1_out, mask2_out, vals, meta,
                                         norms, s);
  return launch_progressive<kValsNone>(W, N, K, Xc, Mc, wanda, mask1_out, mask2_out, nullptr,
                                       nullptr, norms, s);
}

sp24_status sp24_colnorm(const void* Xc, int64_t Mc, int64_t K, double* norms, void* stream) {
  if (!Xc || !norms || Mc < 1 || K < 1) return SP24_ERR_ARG;
  if (K % 8 != 0 || !aligned16(Xc) || !aligned16(norms)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  return launch_colnorm(Xc, Mc, K, norms, as_stream(stream));
}

sp24_status sp24_prune(const void* W, int64_t N, int64_t K, const void* Xc, int64_t Mc,
                       int mode, int n_keep, const uint8_t* mask_in, uint8_t* mask_out,
                       void* workspace, void* stream) {
  if (N < 0 || K < 0 || (mode != SP24_MAGNITUDE && mode != SP24_WANDA) ||
      (n_keep != 2 && n_keep != 3))
    return SP24_ERR_ARG;
  if (N == 0 || K == 0) return SP24_OK;
  if (!W || !mask_out) return SP24_ERR_ARG;
  if (mode == SP24_WANDA && (!Xc || Mc < 1 || !workspace)) return SP24_ERR_ARG;
  if (K % 8 != 0 || !aligned16(W) || !aligned16(mask_out) || (mask_in && !aligned16(mask_in)))
    return SP24_ERR_ALIGN;
  if (mode == SP24_WANDA && (!aligned16(Xc) || !aligned16(workspace))) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  if (mode == SP24_WANDA) {
    return launch_wanda_prune(W, mask_in, mask_out, static_cast<double*>(workspace), N, K, Xc,
                              Mc, n_keep, s);
  }
  return launch_stream<true, false, kValsNone>(W, mask_in, mask_out, nullptr, nullptr, N, K,
                                               n_keep, nullptr, nullptr, s);
}

sp24_status sp24_prune_wanda_noalloc(const void* W, int64_t N, int64_t K, const void* Xc,
                                     int64_t Mc, int n_keep, const uint8_t* mask_in,
                                     uint8_t* mask_out, void* stream) {
  if (N < 0 || K < 0 || (n_keep != 2 && n_keep != 3)) return SP24_ERR_ARG;
  if (K > SP24_NOALLOC_MAX_K) return SP24_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return SP24_OK;
  if (!W || !mask_out || !Xc || Mc < 1) return SP24_ERR_ARG;
  if (K % 8 != 0 || !aligned16(W) || !aligned16(mask_out) || !aligned16(Xc) ||
      (mask_in && !aligned16(mask_in)))
    return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  double* norms = nullptr;
  SP24_TRY(noalloc_norms(&norms));
  return launch_wanda_prune(W, mask_in, mask_out, norms, N, K, Xc, Mc, n_keep,
                            as_stream(stream));
}

sp24_status sp24_wscale(const void* W, const uint8_t* mask, int64_t N, int64_t K,
                        double coverage, float* s_w, void* stream) {
  if (N < 0 || K < 0 || !(coverage > 0.0 && coverage <= 1.0)) return SP24_ERR_ARG;
  if (N == 0) return SP24_OK;
  if (!W || !mask || !s_w) return SP24_ERR_ARG;
  if (K % 8 != 0 || !aligned16(W) || !aligned16(mask) || !aligned16(s_w)) return SP24_ERR_ALIGN;
  if (N > 0x7FFFFFFF) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  return launch_kernel(wscale_kernel, dim3(static_cast<unsigned>((N + 7) / 8)), dim3(256), 0,
                       as_stream(stream), 1, static_cast<const uint16_t*>(W), mask, N, K,
                       coverage, s_w);
}

size_t sp24_act_scale_workspace_bytes(void) { return sizeof(ActScaleWs); }

sp24_status sp24_act_scale(const float* X, int64_t count, double coverage, float* s_x,
                           void* workspace, void* stream) {
  if (!X || !s_x || !workspace || count < 1 || !(coverage > 0.0 && coverage <= 1.0))
    return SP24_ERR_ARG;
  if (count > 0x7FFFFFFFll) return SP24_ERR_ARG;
  if (!aligned16(X) || !aligned16(workspace)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  double rd = ceil(coverage * static_cast<double>(count));
  uint32_t rank = rd < 1.0 ? 1u : static_cast<uint32_t>(rd);
  if (rank > static_cast<uint64_t>(count)) rank = static_cast<uint32_t>(count);
  ActScaleWs* ws = static_cast<ActScaleWs*>(workspace);
  const int64_t nvec = count / 4;
  const int ntail = static_cast<int>(count - nvec * 4);
  if (count >= kActBracketMin) {
    static std::atomic<uint64_t> smem_set{0};   // one bit per device
    const int sel_smem = static_cast<int>(kActSelSmemKeys * 4);
    SP24_TRY(set_smem_once(reinterpret_cast<const void*>(act_bracket_select), sel_smem,
                           smem_set));
    SP24_TRY(launch_kernel(act_sample_load, dim3(kActSampleCtas), dim3(1024), 0, s, 1, X,
                           count, ws));
    SP24_TRY(launch_kernel(act_sample_select, dim3(1), dim3(1024), 0, s, 1, count, rank, ws));
    SP24_TRY(launch_kernel(act_bracket, dim3(grid_for(nvec, 256)), dim3(256), 0, s, 1,
                           reinterpret_cast<const float4*>(X), nvec, X + nvec * 4, ntail, ws));
    SP24_TRY(launch_kernel(act_bracket_select, dim3(1), dim3(1024), sel_smem, s, 1, ws, s_x));
  } else {
    SP24_TRY(launch_kernel(act_scale_init, dim3(1), dim3(256), 0, s, 1, ws, rank));
  }
  const int grid = grid_for(nvec, 256);
  const int shifts[3] = {20, 9, 0};
  const int bitsv[3] = {11, 11, 9};
  uint32_t hi_mask = 0;
  for (int p = 0; p < 3; ++p) {
    SP24_TRY(launch_kernel(act_scale_hist, dim3(grid), dim3(256), 0, s, 1,
                           reinterpret_cast<const float4*>(X), nvec, X + nvec * 4, ntail, ws,
                           shifts[p], bitsv[p], hi_mask, s_x, static_cast<int>(p == 2)));
    hi_mask |= ((1u << bitsv[p]) - 1u) << shifts[p];
  }
  return SP24_OK;
}

sp24_status sp24_fake_quant(const void* W, const uint8_t* mask, int64_t N, int64_t K,
                            const float* s_w, void* W_fq, void* stream) {
  if (N < 0 || K < 0) return SP24_ERR_ARG;
  if (N == 0 || K == 0) return SP24_OK;
  if (!W || !mask || !s_w || !W_fq) return SP24_ERR_ARG;
  if (K % 8 != 0 || !aligned16(W) || !aligned16(W_fq)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  const int64_t kvec = K / 8;
  const int64_t bx = (kvec + 255) / 256;
  const unsigned gx = static_cast<unsigned>(bx < 64 ? bx : 64);
  const unsigned gy = static_cast<unsigned>(N < 65535 ? N : 65535);
  return launch_kernel(fake_quant_kernel, dim3(gx, gy), dim3(256), 0, as_stream(stream), 1,
                       static_cast<const uint4*>(W), mask, s_w, N, kvec,
                       static_cast<uint4*>(W_fq));
}

sp24_status sp24_prune_compress_int8(const void* W, int64_t N, int64_t K, double coverage,
                                    uint8_t* mask_out, float* s_w, void* vals, void* meta,
                                    void* stream) {
  if (N < 0 || K < 0 || !(coverage > 0.0 && coverage <= 1.0)) return SP24_ERR_ARG;
  if (K < 32 || K % 32 != 0) return SP24_ERR_ALIGN;
  if (N == 0) return SP24_OK;
  if (!W || !s_w || !vals || !meta) return SP24_ERR_ARG;
  if (!aligned16(W) || !aligned16(vals) || !aligned16(meta)) return SP24_ERR_ALIGN;
  if (N > (int64_t(1) << 31) || K > (int64_t(1) << 31)) return SP24_ERR_UNSUPPORTED;
  SP24_TRY(check_device());
  const int64_t n_pad = (N + 127) / 128 * 128;   // padding rows of the last tile too
  const dim3 grid(static_cast<unsigned>(n_pad / 4));
  if (K / 8 <= 64 * kInt8HalfVec)
    return launch_kernel(prune_int8_kernel<kInt8HalfVec>, grid, dim3(256), 0, as_stream(stream),
                         1, static_cast<const uint16_t*>(W), N, K, coverage, mask_out, s_w,
                         static_cast<uint32_t*>(vals), static_cast<uint8_t*>(meta));
  return launch_kernel(prune_int8_kernel<0>, grid, dim3(256), 0, as_stream(stream), 1,
                       static_cast<const uint16_t*>(W), N, K, coverage, mask_out, s_w,
                       static_cast<uint32_t*>(vals), static_cast<uint8_t*>(meta));
}

sp24_status sp24_quantize(const float* X, int64_t count, const float* s_x, int8_t* Xq,
                          void* stream) {
  if (count < 0) return SP24_ERR_ARG;
  if (count == 0) return SP24_OK;
  if (!X || !s_x || !Xq) return SP24_ERR_ARG;
  if (!aligned16(X) || !aligned16(Xq)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  const int64_t nvec16 = count / 16;
  if (nvec16 > 0) {
    SP24_TRY(launch_kernel(quantize_kernel, dim3(grid_for(nvec16, 256)), dim3(256), 0, s, 1,
                           reinterpret_cast<const float4*>(X), nvec16, s_x,
                           reinterpret_cast<uint4*>(Xq)));
  }
  const int64_t start = nvec16 * 16;
  if (start < count) {
    SP24_TRY(launch_kernel(quantize_tail, dim3(1), dim3(32), 0, s, 1, X, start, count, s_x, Xq));
  }
  return SP24_OK;
}

sp24_status sp24_compress(const void* W, const uint8_t* mask, int64_t N, int64_t K, int dtype,
                          const float* s_w, void* vals, void* meta, void* stream) {
  if (N < 0 || K < 0 || (dtype != SP24_BF16 && dtype != SP24_INT8)) return SP24_ERR_ARG;
  if (N == 0 || K == 0) return SP24_OK;
  if (!W || !mask || !vals || !meta || (dtype == SP24_INT8 && !s_w)) return SP24_ERR_ARG;
  if (K % (dtype == SP24_BF16 ? 16 : 32) != 0) return SP24_ERR_ALIGN;
  if (!aligned16(W) || !aligned16(mask) || !aligned16(vals) || !aligned16(meta) ||
      (s_w && !aligned16(s_w)))
    return SP24_ERR_ALIGN;
  if ((N + 127) / 128 > 65535) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  if (dtype == SP24_BF16)
    return launch_stream<false, false, kValsBF16>(W, mask, nullptr, nullptr, nullptr, N, K, 2,
                                                  vals, meta, s);
  return launch_stream<false, false, kValsINT8>(W, mask, nullptr, nullptr, s_w, N, K, 2, vals,
                                                meta, s);
}

sp24_status sp24_prune_compress(const void* W, int64_t N, int64_t K, int mode,
                                const double* norms, const uint8_t* mask_in, uint8_t* mask_out,
                                int dtype, const float* s_w, void* vals, void* meta,
                                void* stream) {
  if (N < 0 || K < 0 || (dtype != SP24_BF16 && dtype != SP24_INT8) ||
      (mode != SP24_MAGNITUDE && mode != SP24_WANDA))
    return SP24_ERR_ARG;
  if (N == 0 || K == 0) return SP24_OK;
  if (!W || !vals || !meta || (dtype == SP24_INT8 && !s_w) || (mode == SP24_WANDA && !norms))
    return SP24_ERR_ARG;
  if (K % (dtype == SP24_BF16 ? 16 : 32) != 0) return SP24_ERR_ALIGN;
  if (!aligned16(W) || !aligned16(vals) || !aligned16(meta) || (s_w && !aligned16(s_w)) ||
      (mask_in && !aligned16(mask_in)) || (mask_out && !aligned16(mask_out)) ||
      (norms && !aligned16(norms)))
    return SP24_ERR_ALIGN;
  if ((N + 127) / 128 > 65535) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  const bool wanda = mode == SP24_WANDA;
  if (dtype == SP24_BF16) {
    return wanda ? launch_stream<true, true, kValsBF16>(W, mask_in, mask_out, norms, nullptr, N, K,
                                                        2, vals, meta, s)
                 : launch_stream<true, false, kValsBF16>(W, mask_in, mask_out, nullptr, nullptr, N,
                                                         K, 2, vals, meta, s);
  }
  return wanda ? launch_stream<true, true, kValsINT8>(W, mask_in, mask_out, norms, s_w, N, K, 2,
                                                      vals, meta, s)
               : launch_stream<true, false, kValsINT8>(W, mask_in, mask_out, nullptr, s_w, N, K,
                                                       2, vals, meta, s);
}

}  // extern "C"
