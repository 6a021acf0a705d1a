// Split-K sparse GEMM kernel and its launch.  Included by gemm_sp.cu.
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
#pragma once

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
  //    CTA `split` owns tokens [split*BN/SPLIT, (split+1)*BN/SPLIT) (integer
  //    division: a split that does not divide BN gives some CTAs one token
  //    more).
  const int tok0 = static_cast<int>(split) * BN / SPLIT;
  const int kTokPerCta = (static_cast<int>(split) + 1) * BN / SPLIT - tok0;
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

// ------------------------------------------------------------ host launch
template <int kDtype, int BN, int STAGES, int SPLIT>
sp24_status launch_gemm_cfg(const CUtensorMap& ma, const CUtensorMap& mb, const GemmArgs& a,
                            cudaStream_t s) {
  using C = GemmCfg<kDtype, BN, STAGES>;
  auto kern = gemm_sp_kernel<kDtype, BN, STAGES, SPLIT>;
  static std::atomic<uint64_t> smem_set{0};   // one bit per device
  SP24_TRY(set_smem_once(reinterpret_cast<const void*>(kern), C::kSmemBytes, smem_set));
  const int64_t row_tiles = (a.n + 127) / 128;
  const int64_t tok_tiles = (a.m + BN - 1) / BN;
  if (row_tiles > 65535 || tok_tiles > 65535) return SP24_ERR_UNSUPPORTED;
  return launch_kernel(kern, dim3(SPLIT, static_cast<unsigned>(row_tiles),
                                  static_cast<unsigned>(tok_tiles)),
                       dim3(128), C::kSmemBytes, s, SPLIT, ma, mb, a);
}


}  // namespace sp24
