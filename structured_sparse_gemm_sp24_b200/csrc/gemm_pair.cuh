// Persistent sparse GEMM on CTA pairs (tcgen05 cta_group::2).  Included by
// gemm_sp.cu.
//
// A cluster of two CTAs on two SMs computes 256 (output channels) x BN
// (tokens) tiles.  Each CTA stages its own 128 weight rows (A), its own BN/2
// token rows (B) and its rows' metadata; the even CTA issues one M = 256
// tcgen05.mma.sp per 32 (bf16) / 64 (int8) K-positions that reads both CTAs'
// shared memory and accumulates into both CTAs' tensor memory.  Against a
// 128 x 128 tile on one SM this halves the shared-memory traffic (TMA writes
// plus tensor-core reads) per multiply-add, which is what bounds the
// single-SM version.
//
// Synchronisation:
//  * both CTAs' TMA loads complete on the even CTA's full barrier (its
//    producer arms it with the bytes of both CTAs);
//  * the even CTA's MMA commits arrive on the empty barrier of both CTAs
//    (multicast), so each producer refills its own stage;
//  * tensor-memory full: multicast commit to both epilogues; tensor-memory
//    empty: the even CTA's barrier collects one arrival per epilogue warp of
//    both CTAs.
// Warps: 0 = TMA producer (both CTAs), 1 = MMA issuer (even CTA), 2..9 =
// epilogue (both CTAs; warp 2 also owns the tensor-memory allocation).
#pragma once

namespace sp24 {

template <int kDtype, int BN, int STAGES, int OUTK, int ACC>
struct PairCfg {
  static constexpr int kHalfN = BN / 2;                          // token rows per CTA
  static constexpr int kABytes = 128 * 128;
  static constexpr int kBHalfBytes = kHalfN * 128;               // one K-half of B
  static constexpr int kMetaChunks = kDtype == SP24_BF16 ? 1 : 2;
  static constexpr int kEBytes = 2048 * kMetaChunks;
  static constexpr int kStageBytes = kABytes + 2 * kBHalfBytes + kEBytes;
  static constexpr int kStageStride = (kStageBytes + 1023) / 1024 * 1024;
  static constexpr int kLogicalK = kDtype == SP24_BF16 ? 128 : 256;
  static constexpr int kMmaK = kLogicalK / 4;
  static constexpr int kMetaCols = 4 * kMetaChunks;
  static constexpr int kAcc = ACC;
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

// Instruction descriptor for M = 256 (pair) sparse MMAs.
template <int kDtype, int BN>
__device__ __forceinline__ uint32_t make_idesc_pair(uint32_t id2) {
  const uint32_t c_fmt = kDtype == SP24_BF16 ? 1u : 2u;
  return (id2 & 3u) | (1u << 2) | (c_fmt << 4) | (1u << 7) | (1u << 10) |
         (static_cast<uint32_t>(BN >> 3) << 17) | ((256u >> 4) << 24);
}

template <int kDtype, int BN, int STAGES, int OUTK, int ACC, bool kConv = false>
__global__ void __launch_bounds__(gemm_threads(kConv), 1)
gemm_sp_pair(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
             const __grid_constant__ CUtensorMap tmap_e, const __grid_constant__ CUtensorMap tmap_y,
             const __grid_constant__ CUtensorMap tmap_y16, const PersistArgs args) {
  pdl_launch_dependents();
  using C = PairCfg<kDtype, BN, STAGES, OUTK, ACC>;
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
  const uint32_t rank = cluster_ctarank();            // 0 = even (MMA-issuing) CTA
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int ntiles = args.row_tiles * args.tok_tiles;  // row tiles of 256 here
  const int kchunks = static_cast<int>((args.k + 127) / 128);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < C::kAcc; ++a) {
      mbar_init(&tfull_bar[a], 1);
      mbar_init(&tempty_bar[a], 2 * kEpiWarps);   // epilogue warps of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc_pair(tmem_slot, C::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_prior();   // set-up above overlapped the previous kernel's tail

  if (warp == 0 || (kConv && warp == kConvProducerWarp)) {
    if (lane == 0) {
      // -------------------------------------------------------- producer
      // (the implicit convolution runs two producer warps, each loading every
      // other stage: its token loads take longer to issue)
      const uint32_t pid = warp == 0 ? 0u : 1u;
      prefetch_tmap(&tmap_a);
      prefetch_tmap(&tmap_b);
      prefetch_tmap(&tmap_e);
      uint32_t it = 0;
      for (int tile = pair; tile < ntiles && !*abort_flag; tile += npairs) {
        int prt, tt;
        tile_coords(tile, args, prt, tt);
        const int rt128 = prt * 2 + static_cast<int>(rank);   // this CTA's 128-row tile
        ConvTileRows crow;
        ConvTap ctap{0, 0};
        if constexpr (kConv)
          conv_tile_rows(static_cast<int64_t>(tt) * BN + static_cast<int>(rank) * C::kHalfN, args,
                         crow);
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
          const uint32_t fb = map_peer(smem_u32(&full_bar[s]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2u * C::kStageBytes);
          tma_load_2d_pair(st, &tmap_a, fb, kb * (kDtype == SP24_BF16 ? 64 : 128), rt128 * 128);
          const int kx = kb * C::kLogicalK;
          const int ty = tt * BN + static_cast<int>(rank) * C::kHalfN;
          if constexpr (kConv) {
            conv_load_tokens<C::kHalfN, C::kLogicalK>(
                st + C::kABytes, ctap, crow, args,
                [&](uint8_t* dst, int32_t c, int32_t w, int32_t h, int32_t b) {
                  tma_load_4d_pair(dst, &tmap_b, fb, c, w, h, b);
                });
          } else {
            tma_load_2d_pair(st + C::kABytes, &tmap_b, fb, kx, ty);
            tma_load_2d_pair(st + C::kABytes + C::kBHalfBytes, &tmap_b, fb,
                             kx + C::kLogicalK / 2, ty);
          }
          // metadata map: 8 rows of 256 bytes per 2048-byte chunk
          tma_load_2d_pair(st + C::kABytes + 2 * C::kBHalfBytes, &tmap_e, fb, 0,
                           (rt128 * kchunks + kb * C::kMetaChunks) * 8);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------ MMA issuer
      uint32_t it = 0, j = 0;
      for (int tile = pair; tile < ntiles && !*abort_flag; tile += npairs, ++j) {
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
          for (int c = 0; c < C::kMetaChunks; ++c)
            tc_cp_128x128b_pair(tmem_base + meta_col + 4 * c,
                                smem_desc(e_addr + 2048 * c, 128, 128, kSwizzleNone));
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (q < n_mma) {
              const uint64_t a_desc = smem_desc(a_addr + 32 * q, 0, 1024, kSwizzle128B);
              const uint64_t b_desc = smem_desc(
                  b_addr + (q >> 1) * C::kBHalfBytes + 64 * (q & 1), 0, 1024, kSwizzle128B);
              const uint32_t accumulate = (kb > 0 || q > 0) ? 1u : 0u;
              if constexpr (kDtype == SP24_BF16) {
                tc_mma_sp_pair(d_tmem, a_desc, b_desc, tmem_base + meta_col + (q & ~1),
                               make_idesc_pair<kDtype, BN>(q & 1), accumulate);
              } else {
                tc_mma_sp_i8_pair(d_tmem, a_desc, b_desc, tmem_base + meta_col + 2 * q,
                                  make_idesc_pair<kDtype, BN>(0), accumulate);
              }
            }
          }
          tc_commit_pair_mc(&empty_bar[s], 0x3);   // frees the stage in both CTAs
        }
        tc_commit_pair_mc(&tfull_bar[acc], 0x3);   // both epilogues may drain
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
    for (int tile = pair; tile < ntiles; tile += npairs, ++j) {
      int prt, tt;
      tile_coords(tile, args, prt, tt);
      const int rt128 = prt * 2 + static_cast<int>(rank);
      const uint32_t acc = j % C::kAcc;
      bool ok = true;
      if (lane == 0) ok = !*abort_flag && mbar_wait(&tfull_bar[acc], (j / C::kAcc) & 1u);
      if (!__shfl_sync(0xffffffffu, ok, 0)) { *abort_flag = 1; break; }
      tc_fence_after();
      e.c0 = rt128 * 128 + quad * 32;
      epi_scales<kDtype, OUTK>(e, lane, args.s_w, sx);
      e.tmem = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + acc * BN;
      e.tok0 = static_cast<int64_t>(tt) * BN;
      epilogue_tile<kDtype, OUTK, BN, (ACC == 1)>(e, &tmap_y, &tmap_y16, grp, lane, [&] {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(map_peer(smem_u32(&tempty_bar[acc]), 0));
      });
    }
    if (lane == 0) bulk_wait<0>();
  }

  __syncwarp();
  if (*abort_flag) settle_ns(20000);
  tc_fence_before();
  cluster_sync();          // no CTA leaves while its peer may still signal it
  if (warp == 2) tmem_dealloc_pair(tmem_base, C::kTmemCols);
}

// ------------------------------------------------------------ host launch
template <int kDtype, int BN, int STAGES, int OUTK, int ACC, bool kConv = false>
sp24_status launch_pair(const CUtensorMap& ma, const GemmArgs& g, const void* x, int pairs,
                        cudaStream_t s, const ConvGeom* cg = nullptr) {
  using C = PairCfg<kDtype, BN, STAGES, OUTK, ACC>;
  auto kern = gemm_sp_pair<kDtype, BN, STAGES, OUTK, ACC, kConv>;
  static std::atomic<uint64_t> smem_set{0};   // one bit per device
  SP24_TRY(set_smem_once(reinterpret_cast<const void*>(kern), C::kSmemBytes, smem_set));
  const int el = kDtype == SP24_BF16 ? 2 : 1;
  const CUtensorMapDataType dt =
      kDtype == SP24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  // B: each CTA loads BN/2 token rows (implicit convolution: boxes of whole
  // image rows from the NHWC activations)
  CUtensorMap mb;
  if constexpr (kConv) {
    if (cg == nullptr) return SP24_ERR_ARG;
    SP24_TRY(make_map_nhwc(&mb, x, dt, el, static_cast<uint64_t>(cg->c),
                           static_cast<uint64_t>(cg->w), static_cast<uint64_t>(cg->h),
                           static_cast<uint64_t>(cg->b), static_cast<uint32_t>(128 / el),
                           static_cast<uint32_t>(cg->w), static_cast<uint32_t>(cg->rows)));
  } else {
    SP24_TRY(make_map(&mb, x, dt, el, static_cast<uint64_t>(g.k), static_cast<uint64_t>(g.m),
                      static_cast<uint32_t>(128 / el), static_cast<uint32_t>(C::kHalfN)));
  }
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
  // raster band of 16 row-pair tiles: measured (ncu DRAM bytes per launch) on
  // square 8192^3 and 16384^3 against bands of 3..32, it keeps both the band's
  // weights and the token tiles of a wave in L2 best (16384^3: 10.2 GB read
  // against 18.0 GB with 6)
  int64_t gr = 16;
  gr = group_rows_override(gr);
  gr = gr < 1 ? 1 : (gr > a.row_tiles ? a.row_tiles : gr);
  a.group_rows = static_cast<int>(gr);
  a.y_box = y_box;
  a.conv_h = a.conv_w = a.conv_c = a.conv_rows = a.conv_boxes = 0;
  if constexpr (kConv) {
    a.conv_h = static_cast<int>(cg->h);
    a.conv_w = static_cast<int>(cg->w);
    a.conv_c = static_cast<int>(cg->c);
    a.conv_rows = cg->rows;
    a.conv_boxes = cg->boxes;
    if (cg->boxes * cg->rows * cg->w != C::kHalfN) return SP24_ERR_ARG;
  }
  const int64_t ntiles = static_cast<int64_t>(a.row_tiles) * a.tok_tiles;
  if (ntiles > 0x7FFFFFFF) return SP24_ERR_UNSUPPORTED;
  if (pairs < 1 || pairs > ntiles) return SP24_ERR_ARG;   // the plan sizes the grid
  return launch_kernel(kern, dim3(2 * pairs), dim3(gemm_threads(kConv)), C::kSmemBytes, s, 2, ma,
                       mb, me, my, my16, a);
}

// CTA pairs (clusters of 2) that can be resident at once.  A cluster lives in
// one GPC, so a GPC with an odd number of SMs leaves one out and the count can
// be below SMs / 2; the persistent pair kernels launch exactly this many pairs
// so that no pair waits for another to finish.  Every pair variant holds one
// CTA per SM, so one query (cached per device) serves them all.
inline sp24_status pair_capacity(int* out) {
  static std::atomic<int> cache[64];   // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail("cudaGetDevice", cudaErrorInvalidDevice);
  const int cached = cache[dev & 63].load(std::memory_order_acquire);
  if (cached > 0) {
    *out = cached;
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
  cache[dev & 63].store(n, std::memory_order_release);
  *out = n;
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

}  // namespace sp24
