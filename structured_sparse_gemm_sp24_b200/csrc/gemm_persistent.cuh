// Persistent, warp-specialised sparse GEMM for problems with at least one
// output tile per SM (the tensor-core-bound regime).  Included by gemm_sp.cu.
//
// Same operands, metadata path and MMA issue as the split-K kernel, plus:
//  * one CTA per SM walks a static list of 128 x BN output tiles in a grouped
//    order: GROUP_ROWS weight row tiles are swept across all token tiles
//    before the next group, so one group's compressed weights and the token
//    tiles of a wave stay in L2 (each weight byte is fetched from HBM once);
//  * two tensor-memory accumulators: the MMA warp fills one tile while the
//    epilogue warps drain the other;
//  * eight epilogue warps drain 32 tokens x 32 channels at a time, each with
//    its own staging box and TMA store (the shared epilogue code).
// Warps: 0 = TMA producer, 1 = MMA issuer, 2..9 = epilogue (warp 2 also owns
// the tensor-memory allocation).
#pragma once

namespace sp24 {

template <int kDtype, int BN, int STAGES, int OUTK>
struct PersistCfg {
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBHalfBytes = BN * 128;
  static constexpr int kMetaChunks = kDtype == SP24_BF16 ? 1 : 2;
  static constexpr int kEBytes = 2048 * kMetaChunks;
  static constexpr int kStageBytes = kABytes + 2 * kBHalfBytes + kEBytes;
  static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
  static constexpr int kLogicalK = kDtype == SP24_BF16 ? 128 : 256;
  static constexpr int kMmaK = kLogicalK / 4;
  static constexpr int kMetaCols = 4 * kMetaChunks;
  static constexpr int kAcc = 2;
  static constexpr int kMetaCol0 = kAcc * BN;
  static constexpr int kTmemNeeded = kAcc * BN + 2 * kMetaCols;
  static constexpr int kTmemCols = kTmemNeeded <= 32 ? 32
                                   : kTmemNeeded <= 64 ? 64
                                   : kTmemNeeded <= 128 ? 128
                                   : kTmemNeeded <= 256 ? 256 : 512;
  static constexpr int kOutBytes = EpiOut<OUTK>::kBytes;
  static constexpr int kStagingBytes = EpiOut<OUTK>::kStagingBytes;  // all epilogue warps
  static constexpr int kRingBytes = STAGES * kStageStride;
  static constexpr int kSmemBytes = kRingBytes + kStagingBytes + 1024 + 256;
  static_assert(kTmemNeeded <= 512, "tensor memory overflow");
  static_assert(BN % 16 == 0 && BN >= 64 && BN <= 256, "BN");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct PersistArgs {
  const uint8_t* meta;
  const float* s_x;
  const float* s_w;
  const float* s_y;
  int64_t m, n, k;
  int kblocks;       // K stages per tile
  int row_tiles;     // ceil(N / 128)
  int tok_tiles;     // ceil(M / BN)
  int group_rows;    // raster group height (row tiles)
  int y_box;         // channels per epilogue store box: min(32, N)
  // implicit 3x3 convolution (pair kernel with kConv): NHWC image sizes and
  // the token loads (boxes of conv_rows image rows of conv_w pixels each)
  int conv_h, conv_w, conv_c;
  int conv_rows;     // image rows per TMA box
  int conv_boxes;    // boxes per K-half of a CTA's token rows
};

// SP24_GEMM_GROUP_ROWS = n > 0: raster group height in weight row tiles
// (tuning override of the persistent kernels; results do not depend on it).
inline int64_t group_rows_override(int64_t gr) {
  const char* e = std::getenv("SP24_GEMM_GROUP_ROWS");
  if (!e) return gr;
  const long v = std::atol(e);
  return v > 0 ? static_cast<int64_t>(v) : gr;
}

// Geometry of the implicit 3x3 convolution (NHWC X of b x h x w x c); its
// launches read the token operand through a 4D map of X instead of a 2D map.
struct ConvGeom {
  int64_t b, h, w, c;
  int rows;    // image rows per TMA box
  int boxes;   // boxes per K-half of the tokens one CTA loads
};

// Linear tile index -> (row tile, token tile) in the grouped order.
__device__ __forceinline__ void tile_coords(int t, const PersistArgs& a, int& rt, int& tt) {
  const int per_group = a.group_rows * a.tok_tiles;
  const int g = t / per_group;
  const int r = t - g * per_group;
  int rows = a.row_tiles - g * a.group_rows;
  rows = rows < a.group_rows ? rows : a.group_rows;
  rt = g * a.group_rows + r % rows;
  tt = r / rows;
}

// Token operand of the implicit 3x3 convolution (stride 1, padding 1, NHWC):
// the tile's tokens are whole image rows, so for k-block kb the K-half h
// (kLogicalK / 2 consecutive K positions, all in one tap because C * element
// bytes is a multiple of 128) is the image shifted by the tap, read through
// the 4D map (c, w, h, b) at (c0, kw - 1, row + kh - 1, b); the zero fill
// outside the image is the padding.  Half-k-blocks past K = 9 C read a
// channel coordinate past C (all zero).  Each box is conv_rows rows x
// conv_w pixels (a multiple of 8 rows of 128 bytes, so every box starts on a
// 1024-byte boundary of the swizzled tile).  kTok: tokens of the tile this
// CTA loads (BN / 2 in the pair kernel, BN in the single-SM kernel).
//
// The producer is one thread and the loads are on its critical path, so the
// per-box (image, row) pairs are formed once per tile with 32-bit divisions
// and the (tap, channel) of each K-half is advanced without dividing.
constexpr int kConvMaxBoxes = 16;

struct ConvTileRows {
  int32_t b[kConvMaxBoxes];
  int32_t row[kConvMaxBoxes];
};

__device__ __forceinline__ void conv_tile_rows(int64_t tok0, const PersistArgs& a,
                                               ConvTileRows& t) {
  const uint32_t hw = static_cast<uint32_t>(a.conv_h) * static_cast<uint32_t>(a.conv_w);
  const uint32_t box_tok = static_cast<uint32_t>(a.conv_w * a.conv_rows);
  // tok0 < M < 2^31; tokens past M fall in images >= B (zero fill)
#pragma unroll
  for (int i = 0; i < kConvMaxBoxes; ++i) {
    if (i < a.conv_boxes) {
      const uint32_t p = static_cast<uint32_t>(tok0) + static_cast<uint32_t>(i) * box_tok;
      const uint32_t b = p / hw;
      t.b[i] = static_cast<int32_t>(b);
      t.row[i] = static_cast<int32_t>((p - b * hw) / static_cast<uint32_t>(a.conv_w));
    }
  }
}

// (tap, c0) of the K-half that starts at K position (tap * C + c0); advance()
// moves to the next K-half.
struct ConvTap {
  int tap, c0;
  __device__ __forceinline__ void advance(int half_k, int c) {
    c0 += half_k;
    if (c0 >= c) { c0 = 0; ++tap; }
  }
};

// `load(dst, c, w, h, b)` issues one box load (the pair kernel completes it
// on the even CTA's barrier, the single-SM kernel on its own).
template <int kTok, int kLogicalK, class Load>
__device__ __forceinline__ void conv_load_tokens(uint8_t* dst, ConvTap& tp, const ConvTileRows& t,
                                                 const PersistArgs& a, Load&& load) {
  const int box_bytes = a.conv_w * a.conv_rows * 128;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const bool past = tp.tap >= 9;
    const int kh = past ? 1 : tp.tap / 3;
    const int kw = past ? 1 : tp.tap - 3 * (tp.tap / 3);
    const int c0 = past ? a.conv_c : tp.c0;
#pragma unroll
    for (int i = 0; i < kConvMaxBoxes; ++i) {
      if (i < a.conv_boxes)
        load(dst + half * (kTok * 128) + i * box_bytes, c0, kw - 1, t.row[i] + kh - 1, t.b[i]);
    }
    tp.advance(kLogicalK / 2, a.conv_c);
  }
}

template <int kDtype, int BN, int STAGES, int OUTK, bool kConv = false>
__global__ void __launch_bounds__(gemm_threads(kConv), 1)
gemm_sp_persistent(const __grid_constant__ CUtensorMap tmap_a,
                   const __grid_constant__ CUtensorMap tmap_b,
                   const __grid_constant__ CUtensorMap tmap_y,
                   const __grid_constant__ CUtensorMap tmap_y16, const PersistArgs args) {
  pdl_launch_dependents();
  using C = PersistCfg<kDtype, BN, STAGES, OUTK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* staging = smem + C::kRingBytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(staging + C::kStagingBytes);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* tfull_bar = empty_bar + STAGES;
  uint64_t* tempty_bar = tfull_bar + C::kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty_bar + C::kAcc);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int ntiles = args.row_tiles * args.tok_tiles;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < C::kAcc; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], kEpiWarps);   // one arrival per epilogue warp
    }
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
  pdl_wait_prior();   // set-up above overlapped the previous kernel's tail
  const int kchunks = static_cast<int>((args.k + 127) / 128);

  if (warp == 0 || (kConv && warp == kConvProducerWarp)) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      // (the implicit convolution runs two producer warps, each loading every
      // other stage: its token loads take longer to issue)
      const uint32_t pid = warp == 0 ? 0u : 1u;
      prefetch_tmap(&tmap_a);
      prefetch_tmap(&tmap_b);
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x) {
        int rt, tt;
        tile_coords(tile, args, rt, tt);
        const uint8_t* meta_tile = args.meta + static_cast<int64_t>(rt) * kchunks * 2048;
        ConvTileRows crow;
        ConvTap ctap{0, 0};
        if constexpr (kConv) conv_tile_rows(static_cast<int64_t>(tt) * BN, args, crow);
        for (int kb = 0; kb < args.kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          if (kConv && (it & 1u) != pid) {   // the other producer's stage
            if constexpr (kConv) {
              ctap.advance(C::kLogicalK / 2, args.conv_c);
              ctap.advance(C::kLogicalK / 2, args.conv_c);
            }
            continue;
          }
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&empty_bar[s], ph ^ 1u)) { *abort_flag = 1; break; }
          uint8_t* st = smem + s * C::kStageStride;
          int chunks = C::kMetaChunks;
          if (kDtype == SP24_INT8 && 2 * kb + 1 >= kchunks) chunks = 1;
          mbar_arrive_expect_tx(&full_bar[s], C::kABytes + 2 * C::kBHalfBytes + 2048 * chunks);
          tma_load_2d(st, &tmap_a, &full_bar[s], kb * (kDtype == SP24_BF16 ? 64 : 128), rt * 128);
          const int kx = kb * C::kLogicalK;
          if constexpr (kConv) {
            conv_load_tokens<BN, C::kLogicalK>(
                st + C::kABytes, ctap, crow, args,
                [&](uint8_t* dst, int32_t c, int32_t w, int32_t h, int32_t b) {
                  tma_load_4d(dst, &tmap_b, &full_bar[s], c, w, h, b);
                });
          } else {
            tma_load_2d(st + C::kABytes, &tmap_b, &full_bar[s], kx, tt * BN);
            tma_load_2d(st + C::kABytes + C::kBHalfBytes, &tmap_b, &full_bar[s],
                        kx + C::kLogicalK / 2, tt * BN);
          }
          bulk_load(st + C::kABytes + 2 * C::kBHalfBytes,
                    meta_tile + static_cast<int64_t>(kb * C::kMetaChunks) * 2048,
                    2048u * chunks, &full_bar[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      uint32_t it = 0, j = 0;
      for (int tile = blockIdx.x; tile < ntiles && !*abort_flag; tile += gridDim.x, ++j) {
        const uint32_t acc = j % C::kAcc;
        if (!mbar_wait(&tempty_bar[acc], ((j / C::kAcc) & 1u) ^ 1u)) { *abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        bool aborted = false;
        for (int kb = 0; kb < args.kblocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1u;
          if (!mbar_wait(&full_bar[s], ph)) { *abort_flag = 1; aborted = true; break; }
          tc_fence_after();
          uint8_t* st = smem + s * C::kStageStride;
          const uint32_t a_addr = smem_u32(st);
          const uint32_t b_addr = smem_u32(st + C::kABytes);
          const uint32_t e_addr = smem_u32(st + C::kABytes + 2 * C::kBHalfBytes);
          const uint32_t meta_col = C::kMetaCol0 + (it & 1u) * C::kMetaCols;
          const int64_t k_left = args.k - static_cast<int64_t>(kb) * C::kLogicalK;
          int n_mma = static_cast<int>((k_left + C::kMmaK - 1) / C::kMmaK);
          n_mma = n_mma > 4 ? 4 : n_mma;
          const int chunks = kDtype == SP24_BF16 ? 1 : (n_mma > 2 ? 2 : 1);
          for (int c = 0; c < chunks; ++c)
            tc_cp_128x128b(tmem_base + meta_col + 4 * c,
                           smem_desc(e_addr + 2048 * c, 128, 128, kSwizzleNone));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q < n_mma) {
              const uint64_t a_desc = smem_desc(a_addr + 32 * q, 0, 1024, kSwizzle128B);
              const uint64_t b_desc = smem_desc(
                  b_addr + (q >> 1) * C::kBHalfBytes + 64 * (q & 1), 0, 1024, kSwizzle128B);
              const uint32_t accumulate = (kb > 0 || q > 0) ? 1u : 0u;
              if constexpr (kDtype == SP24_BF16) {
                tc_mma_sp(d_tmem, a_desc, b_desc, tmem_base + meta_col + (q & ~1),
                          make_idesc<kDtype, BN>(q & 1), accumulate);
              } else {
                tc_mma_sp_i8(d_tmem, a_desc, b_desc, tmem_base + meta_col + 2 * q,
                             make_idesc<kDtype, BN>(0), accumulate);
              }
            }
          }
          tc_commit(&empty_bar[s]);
        }
        tc_commit(&tfull_bar[acc]);   // accumulator of this tile complete (or abandoned)
        if (aborted) break;
      }
    }
  } else if (warp < 2 + kEpiWarps) {
    // --------------------------------------------------------- epilogue
    const int ew = warp - 2;                 // 0..7
    const int grp = ew >> 2;                 // which chunks of a tile (even / odd)
    const int quad = warp & 3;               // tensor-memory lane quadrant of this warp
    const float sx = (kDtype == SP24_INT8 && OUTK != SP24_OUT_INT32) ? *args.s_x : 1.0f;
    EpiWarp e;
    e.m = args.m;
    e.n = args.n;
    e.cbox = args.y_box;
    e.vec = OUTK == SP24_OUT_BF16 && args.y_box == kEpiBox;
    e.stg = staging + ew * EpiOut<OUTK>::kWarpBytes;
    e.sy = (kDtype == SP24_INT8 && OUTK == SP24_OUT_INT8) ? *args.s_y : 1.0f;
    uint32_t j = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++j) {
      int rt, tt;
      tile_coords(tile, args, rt, tt);
      const uint32_t acc = j % C::kAcc;
      bool ok = true;
      if (lane == 0) ok = !*abort_flag && mbar_wait(&tfull_bar[acc], (j / C::kAcc) & 1u);
      if (!__shfl_sync(0xffffffffu, ok, 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      e.c0 = rt * 128 + quad * 32;
      epi_scales<kDtype, OUTK>(e, lane, args.s_w, sx);
      e.tmem = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      e.tok0 = static_cast<int64_t>(tt) * BN;
      epilogue_tile<kDtype, OUTK, BN, false>(e, &tmap_y, &tmap_y16, grp, lane, [&] {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty_bar[acc]);   // accumulator drained
      });
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  if (*abort_flag) settle_ns(20000);
  tc_fence_before();
  __syncthreads();
  if (warp == 2) tmem_dealloc(tmem_base, C::kTmemCols);
}

// ------------------------------------------------------------ host launch
template <int kDtype, int BN, int STAGES, int OUTK, bool kConv = false>
sp24_status launch_persistent(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& g,
                              cudaStream_t s, const ConvGeom* cg = nullptr) {
  using C = PersistCfg<kDtype, BN, STAGES, OUTK>;
  auto kern = gemm_sp_persistent<kDtype, BN, STAGES, OUTK, kConv>;
  static std::atomic<uint64_t> smem_set{0};   // one bit per device
  SP24_TRY(set_smem_once(reinterpret_cast<const void*>(kern), C::kSmemBytes, smem_set));
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
  a.row_tiles = static_cast<int>((g.n + 127) / 128);
  a.tok_tiles = static_cast<int>((g.m + BN - 1) / BN);
  // raster group: as many weight row tiles as fit ~24 MB of compressed weights
  const int64_t row_tile_bytes = 128 * (g.k / 2) * (kDtype == SP24_BF16 ? 2 : 1);
  int64_t gr = (int64_t(24) << 20) / (row_tile_bytes > 0 ? row_tile_bytes : 1);
  gr = group_rows_override(gr);
  gr = gr < 1 ? 1 : (gr > a.row_tiles ? a.row_tiles : gr);
  a.group_rows = static_cast<int>(gr);
  a.y_box = y_box;
  a.conv_h = a.conv_w = a.conv_c = a.conv_rows = a.conv_boxes = 0;
  if constexpr (kConv) {
    if (cg == nullptr || cg->boxes * cg->rows * cg->w != BN) return SP24_ERR_ARG;
    a.conv_h = static_cast<int>(cg->h);
    a.conv_w = static_cast<int>(cg->w);
    a.conv_c = static_cast<int>(cg->c);
    a.conv_rows = cg->rows;
    a.conv_boxes = cg->boxes;
  }
  const int64_t ntiles = static_cast<int64_t>(a.row_tiles) * a.tok_tiles;
  if (ntiles > 0x7FFFFFFF) return SP24_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(ntiles < sm_count() ? ntiles : sm_count());
  return launch_kernel(kern, dim3(grid), dim3(gemm_threads(kConv)), C::kSmemBytes, s, 1, ma, mb, my,
                       my16, a);
}


}  // namespace sp24
