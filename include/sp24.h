/*
 * sp24.h -- C ABI of libsp24: 2:4 fine-grained structured sparsity on B200.
 *
 * Three verbs, each an asynchronous launch on a caller stream:
 *   prune    W (+ calibration rows)          -> keep mask     (N:4, n_keep of 4)
 *   compress W + mask (+ INT8 scales)        -> values + metadata (tcgen05 operand layout)
 *   gemm     X, values, metadata (+ scales)  -> Y = X * W'^T
 * plus the INT8 calibration helpers (per-channel / per-tensor scales,
 * activation quantisation), the channel permutation search that may precede
 * pruning, and status queries.
 *
 * Sources ("pages") are cited by title and section:
 *   [Ampere-sparsity] NVIDIA x Tencent MLPD article on Ampere fine-grained
 *       structured sparsity (nvidia.zhidx.com): 2:4 pattern and compressed
 *       format (Figure 1), progressive sparsity (Figures 3-4), "PTQ and QAT".
 *   [Wanda-2:4] "Structured Pruning: 2:4 sparse inference with the Wanda
 *       algorithm" (zyxy.net), sections 1.3, 2.1, 2.2.
 *   [Sparse-accel forum] oeforum.com post on sparse acceleration (2-bit
 *       metadata, offline conversion, INT8 x 2:4).
 *   [Orin ch.7] "Chapter 7: 2:4 Structured Sparsity" (Orin NN design book),
 *       sections 2.1 (worked example), 2.3 (alignment), 6.1 (every 1x4 block
 *       must be valid or the sparse path silently falls back), 6.2 (padding).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers named W, X, Xc, A*, mask*, vals, meta, norms, perm, s_*, Y and workspace are
 *   DEVICE pointers owned by the caller; the library never allocates, frees or
 *   keeps them.  Matrices are row-major and densely packed (row stride = number
 *   of columns).  Every device pointer must be 16-byte aligned (cudaMalloc
 *   gives 256) or the call returns SP24_ERR_ALIGN.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Every call only enqueues work; it does not synchronise, except
 *   sp24_permute_search, which says so.
 * - Argument, size and alignment errors are detected on the host before any
 *   launch and returned synchronously; nothing is enqueued in that case.
 * - Errors found on the device (a group that does not keep exactly two
 *   positions, a bounded wait that gave up) are recorded in a per-device
 *   status word and reported by sp24_device_status().
 * - bf16 means IEEE-754 binary32 truncated to its top 16 bits (bfloat16); the
 *   library reads inputs as bit patterns and assumes finite values.
 * - Weight layout: W[N][K], N = output channels, K = input channels; groups of
 *   4 run along K ([Orin ch.7] 2.1).  A 1x1 convolution over NHWC activations
 *   is the same GEMM with M = batch*H*W and K = C_in ([Orin ch.7] 2.2).
 */
#ifndef SP24_H_
#define SP24_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sp24_status {
    SP24_OK = 0,
    SP24_ERR_ARG = 1,         /* null pointer, negative size, unknown enum value */
    SP24_ERR_ALIGN = 2,       /* a size or pointer breaks an alignment rule */
    SP24_ERR_PATTERN = 3,     /* a group of 4 does not keep exactly two positions */
    SP24_ERR_CUDA = 4,        /* a CUDA runtime call failed */
    SP24_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up */
    SP24_ERR_UNSUPPORTED = 6, /* no sm_100 device, or a combination not provided */
    SP24_ERR_INDEX = 7        /* a permutation entry lies outside [0, K) */
} sp24_status;

/* scoring modes for sp24_prune */
enum { SP24_MAGNITUDE = 0, SP24_WANDA = 1 };
/* value types of the compressed weight and of X in sp24_gemm */
enum { SP24_BF16 = 0, SP24_INT8 = 1 };
/* output kinds of sp24_gemm */
enum { SP24_OUT_BF16 = 0, SP24_OUT_INT32 = 1, SP24_OUT_INT8 = 2 };

/* ------------------------------------------------------------------ sizes */

/* Bytes of a keep mask for W[N][K]: one nibble per group of 4 (bit p set when
 * position p is kept), group 2b in the low nibble of byte b; N*K/8.
 * K must be a multiple of 8.  Returns 0 for invalid sizes. */
size_t sp24_mask_bytes(int64_t N, int64_t K);

/* Bytes of the compressed values: N rows of K/2 kept values, in ascending
 * position order within each group ([Ampere-sparsity] Figure 1:
 * only the nonzeros are stored, 50 % of the value bytes).
 * dtype SP24_BF16 -> 2 bytes each, SP24_INT8 -> 1 byte each. */
size_t sp24_vals_bytes(int64_t N, int64_t K, int dtype);

/* Bytes of the metadata: 2 bits per kept value = 4 bits per group
 * ([Sparse-accel forum]; [Orin ch.7] 2.1 "Metadata (2-bit)"), stored in the
 * tcgen05.mma.sp operand layout: chunks of 128 rows x 128 K-positions
 * (2048 bytes), N rounded up to 128 and K rounded up to 128.
 * The layout depends on dtype but the size does not. */
size_t sp24_meta_bytes(int64_t N, int64_t K);

/* Scratch bytes sp24_prune needs for `mode`: 8*K (float64 column norms) for
 * SP24_WANDA, 0 for SP24_MAGNITUDE. */
size_t sp24_prune_workspace_bytes(int64_t K, int mode);

/* ------------------------------------------------------------- pruning */

/* Wanda activation statistic ([Wanda-2:4] 2.1): norms[j] = sqrt(sum_t Xc[t][j]^2)
 * over the Mc calibration rows, float64, summed sequentially in t (each
 * square of a bf16 value is exact in float64; one rounding per addition).
 * Xc: bf16 [Mc][K].  norms: float64 [K].  Mc >= 1, K >= 1, K % 8 == 0. */
sp24_status sp24_colnorm(const void* Xc, int64_t Mc, int64_t K, double* norms,
                         void* stream);

/* N:4 pruning along K ([Wanda-2:4] 1.3 and 2.2; [Orin ch.7] 2.1 Step 1):
 * within each group of 4 consecutive weights of a row, keep the n_keep
 * positions of largest score; position p is kept iff fewer than n_keep others
 * beat it, q beating p when s_q > s_p or (s_q == s_p and q < p).
 *   mode SP24_MAGNITUDE: s = |w|
 *   mode SP24_WANDA:     s = |w| * norms[j] in float64, norms from Xc as in
 *                        sp24_colnorm, computed into `workspace`
 * n_keep = 3 is the 25 % stage of progressive sparsity, n_keep = 2 the 50 %
 * stage ([Ampere-sparsity] Figure 4).  With mask_in != NULL the weights
 * dropped by mask_in score 0 (the second stage recomputes the mask on the
 * remaining weights).
 *   W: bf16 [N][K].  Xc: bf16 [Mc][K] (SP24_WANDA only, else ignored).
 *   mask_in (nullable), mask_out: sp24_mask_bytes(N, K) bytes.
 *   workspace: sp24_prune_workspace_bytes(K, mode) bytes (NULL if 0).  For
 *              SP24_WANDA it holds the float64 column norms [K] afterwards,
 *              ready to pass as `norms` to sp24_prune_compress.
 * Rules: N >= 0, K % 8 == 0, n_keep in {2, 3}; Mc >= 1 for SP24_WANDA. */
sp24_status sp24_prune(const void* W, int64_t N, int64_t K, const void* Xc,
                       int64_t Mc, int mode, int n_keep, const uint8_t* mask_in,
                       uint8_t* mask_out, void* workspace, void* stream);

/* ------------------------------------------------- channel permutation */

/* Largest K accepted by the permutation search (its gain table is K x K
 * int64). */
#define SP24_PERMUTE_MAX_K 65536

/* Outcome of sp24_permute_search (host struct). */
typedef struct sp24_permute_result_t {
    int64_t swaps;        /* exchanges made */
    int64_t kept_before;  /* kept score of the identity order (integer scores) */
    int64_t kept_after;   /* kept score of the returned order */
} sp24_permute_result_t;

/* Scratch bytes of sp24_permute_search: 8*N*K + 8*K*K + O(N + K); 0 for
 * arguments the search rejects. */
size_t sp24_permute_workspace_bytes(int64_t N, int64_t K);

/* Channel permutation search before masking ([Orin ch.7] 3.1 workflow step 2
 * and 6.3: choose an order of the input channels so that large weights share
 * groups of 4 before the mask is made).  The pages give the goal only; this
 * library reads it as:
 *   objective  kept score = over every row and every group of 4 consecutive
 *              positions of W[:, perm], the sum of the n_keep largest scores;
 *   scores     s = |w| (norms == NULL) or |w| * norms[j] (float64, the
 *              sp24_prune Wanda score), a score that is not a finite positive
 *              number counting as 0; compared as the integers
 *              q = rint(s / s_max * 2^24) (float64 divide, half to even), so
 *              every comparison below is exact;
 *   search     greedy exchange: starting from the identity, repeatedly swap
 *              the two channels in different groups whose swap raises the
 *              kept score most (ties: smallest lower channel index, then
 *              smallest upper index); stop when no swap raises it or after
 *              max_swaps swaps.
 *   W: bf16 [N][K].  norms: float64 [K] or NULL.
 *   perm: int32 [K] (device, written): position j of the new order holds
 *         channel perm[j]; apply it with sp24_permute_columns to W and to
 *         the matching columns of X (Y is unchanged), then prune as usual.
 *   workspace: sp24_permute_workspace_bytes(N, K) bytes (workspace_bytes
 *         says how many the caller passes).
 *   result: host struct, nullable.
 * The call BLOCKS the calling thread: it synchronises `stream` between
 * batches of steps to learn whether the search has stopped.
 * Rules: N >= 1, 4 <= K <= SP24_PERMUTE_MAX_K, K % 4 == 0, n_keep in {2, 3},
 * max_swaps >= 0; norms, if given, >= 0 (as sp24_colnorm writes them). */
sp24_status sp24_permute_search(const void* W, int64_t N, int64_t K, const double* norms,
                                int n_keep, int64_t max_swaps, int32_t* perm,
                                void* workspace, size_t workspace_bytes,
                                sp24_permute_result_t* result, void* stream);

/* Column gather that applies a channel order: A_out[r][j] = A[r][perm[j]] for
 * a row-major [rows][K] matrix of elem_bytes-byte elements (1, 2 or 4: int8,
 * bf16, float32).  A and A_out must not overlap.  An entry of perm outside
 * [0, K) writes 0 and records SP24_ERR_INDEX in the device status word. */
sp24_status sp24_permute_columns(const void* A, int64_t rows, int64_t K, int elem_bytes,
                                 const int32_t* perm, void* A_out, void* stream);

/* --------------------------------------------------------- INT8 scales */

/* Per-output-channel weight scale ([Ampere-sparsity] "PTQ and QAT": the scale
 * covers `coverage` (0.9999) of the values): t_n = the r-th smallest |W[n][k]|
 * over the c kept positions of row n, r = max(1, ceil(coverage * c)) computed
 * in IEEE double; s_w[n] = float(t_n) / 127.0f (float32 divide), or 1 when
 * t_n == 0.  For c <= 9999 and coverage 0.9999 this is the row maximum.
 *   W: bf16 [N][K].  mask: sp24_mask_bytes(N, K) bytes.  s_w: float32 [N].
 * Rules: K % 8 == 0, 0 < coverage <= 1. */
sp24_status sp24_wscale(const void* W, const uint8_t* mask, int64_t N, int64_t K,
                        double coverage, float* s_w, void* stream);

/* Per-tensor activation scale: t = the r-th smallest |X[i]| over all `count`
 * float32 values, r = max(1, ceil(coverage * count)) in IEEE double;
 * *s_x = t / 127.0f (float32), or 1 when t == 0.  Exact order statistic of the
 * float32 bit patterns: a bracket from a stratified sample is checked exactly
 * against the counts of one pass over X and the answer selected among the
 * values inside it; when the check fails (central coverages, heavy ties)
 * three exact radix passes decide.
 *   X: float32 [count].  s_x: one float32 (device).
 *   workspace: sp24_act_scale_workspace_bytes() bytes.
 * Rules: count >= 1, 0 < coverage <= 1. */
size_t sp24_act_scale_workspace_bytes(void);
sp24_status sp24_act_scale(const float* X, int64_t count, double coverage,
                           float* s_x, void* workspace, void* stream);

/* Symmetric quantisation: Xq[i] = clamp(rint(X[i] / *s_x), -127, 127) with an
 * IEEE float32 divide and round-half-to-even.
 *   X: float32 [count].  s_x: one float32 (device).  Xq: int8 [count]. */
sp24_status sp24_quantize(const float* X, int64_t count, const float* s_x,
                          int8_t* Xq, void* stream);

/* Forward fake-quantisation of the masked weights for quantisation-aware
 * training ([Ampere-sparsity] "PTQ and QAT": the forward pass quantises the
 * weights to int8 and dequantises them back to floating point; the STE
 * backward pass and training are not part of this library):
 *   kept position:    W_fq = bf16_rne(float(q) * s_w[n]),
 *                     q = clamp(rint(W / s_w[n]), -127, 127), float32 divide,
 *                     round half to even (the code sp24_compress(SP24_INT8)
 *                     stores for the same W, mask and s_w);
 *   dropped position: W_fq = +0.
 *   W, W_fq: bf16 [N][K].  mask: sp24_mask_bytes(N, K) bytes.  s_w: float32
 *   [N] (from sp24_wscale).
 * Rules: N >= 0, K % 8 == 0; W and W_fq 16-byte aligned. */
sp24_status sp24_fake_quant(const void* W, const uint8_t* mask, int64_t N, int64_t K,
                            const float* s_w, void* W_fq, void* stream);


/* ---------------------------------------------------------- compression */

/* Compression ([Ampere-sparsity] Figure 1; [Orin ch.7] 2.1 Step 2): for each
 * group with kept positions lo < hi, vals gets W[lo] then W[hi] and the
 * metadata records the two 2-bit positions.
 *   dtype SP24_BF16: vals bf16 [N][K/2] (the weights' own bits).
 *   dtype SP24_INT8: vals int8 [N][K/2], q = clamp(rint(W / s_w[n]), -127, 127)
 *                    with a float32 divide (s_w from sp24_wscale).
 *   meta: sp24_meta_bytes(N, K) bytes in the operand layout of
 *         tcgen05.mma.sp for `dtype` (opaque to callers; rows >= N and
 *         positions >= K are filled with a valid pattern over zero values).
 * A group whose mask nibble does not have exactly two bits set is a pattern
 * error ([Orin ch.7] 6.1): it is reported by sp24_device_status() as
 * SP24_ERR_PATTERN (never silently treated as dense); its outputs are
 * unspecified.
 * Rules: K % 8 == 0 (SP24_BF16: K % 16 == 0; SP24_INT8: K % 32 == 0, so that
 * value rows stay 16-byte aligned); s_w required for SP24_INT8. */
sp24_status sp24_compress(const void* W, const uint8_t* mask, int64_t N, int64_t K,
                          int dtype, const float* s_w, void* vals, void* meta,
                          void* stream);

/* Fused prune + compress in one pass over W: the mask of sp24_prune (with
 * n_keep = 2) and the outputs of sp24_compress.  mask_out may be NULL.
 * norms: float64 [K] from sp24_colnorm for SP24_WANDA, else NULL. */
sp24_status sp24_prune_compress(const void* W, int64_t N, int64_t K, int mode,
                                const double* norms, const uint8_t* mask_in,
                                uint8_t* mask_out, int dtype, const float* s_w,
                                void* vals, void* meta, void* stream);

/* INT8 weight conversion in one pass over W ([Ampere-sparsity] "PTQ and QAT"
 * for the per-channel scale at `coverage`; [Orin ch.7] 2.1 Steps 1-2 for the
 * magnitude 2:4 mask and the compressed stream): the outputs of
 *   sp24_prune(W, mode = SP24_MAGNITUDE, n_keep = 2)          -> mask_out,
 *   sp24_wscale(W, that mask, coverage)                      -> s_w,
 *   sp24_compress(W, that mask, SP24_INT8, s_w)              -> vals, meta,
 * bit for bit, from one kernel instead of three passes over W.
 *   W: bf16 [N][K].  mask_out: sp24_mask_bytes(N, K) bytes or NULL.
 *   s_w: float32 [N].  vals: int8 [N][K/2].  meta: sp24_meta_bytes(N, K).
 * Rules: N >= 0, K >= 32, K % 32 == 0, 0 < coverage <= 1; W, vals and meta
 * 16-byte aligned. */
sp24_status sp24_prune_compress_int8(const void* W, int64_t N, int64_t K, double coverage,
                                     uint8_t* mask_out, float* s_w, void* vals, void* meta,
                                     void* stream);

/* Progressive pruning in one pass ([Ampere-sparsity] Figure 4: the 25 %
 * stage keeps 3 of every 4 weights, the 50 % stage keeps 2 of 4 of the
 * weights the first stage kept).  With no fine-tuning between the stages both
 * masks come from the same weights, so one pass over W computes
 *   mask1_out = the mask of sp24_prune(W, ..., n_keep = 3, mask_in = NULL)
 *   mask2_out = the mask of sp24_prune(W, ..., n_keep = 2, mask_in = mask1)
 * and, when vals and meta are given, the bf16 compression of W under mask2
 * (the outputs of sp24_compress(W, mask2, SP24_BF16, ...)).
 *   W: bf16 [N][K].  Xc, Mc, mode, workspace: as sp24_prune (for SP24_WANDA
 *   the workspace holds the float64 column norms afterwards).
 *   mask1_out, mask2_out: sp24_mask_bytes(N, K) bytes each, nullable.
 *   vals, meta: both NULL (masks only) or both given (bf16 values [N][K/2],
 *   sp24_meta_bytes(N, K) bytes of metadata).
 * Rules: N >= 0, K % 8 == 0 (K % 16 == 0 with compression), at least one
 * output; Mc >= 1 and a workspace for SP24_WANDA. */
sp24_status sp24_prune_progressive(const void* W, int64_t N, int64_t K, const void* Xc,
                                   int64_t Mc, int mode, uint8_t* mask1_out,
                                   uint8_t* mask2_out, void* vals, void* meta,
                                   void* workspace, void* stream);

/* ----------------------------------------------------------- sparse GEMM */

/* Y = X * W'^T with W' the 2:4 weight given by (vals, meta) ([Orin ch.7] 2.1
 * Step 3: only the kept weights are multiplied, each with the activation its
 * 2-bit position selects; [Sparse-accel forum]: INT8 x 2:4).
 *   dtype SP24_BF16: X bf16 [M][K]; fp32 accumulation; out_kind SP24_OUT_BF16
 *       writes Y bf16 [M][N] = rne(acc).  s_x, s_w, s_y ignored (may be NULL).
 *   dtype SP24_INT8: X int8 [M][K] (from sp24_quantize); int32 accumulation,
 *       exact.  out_kind SP24_OUT_INT32: Y int32 [M][N] = acc.
 *       SP24_OUT_BF16: Y bf16 = rne(float(acc) * (s_x * s_w[n])), each step
 *       float32 round-to-nearest, in that order.
 *       SP24_OUT_INT8: Y int8 = clamp(rint((float(acc) * (s_x * s_w[n])) / s_y),
 *       -127, 127), float32 divide.
 *       s_x, s_y: one float32 each (device); s_w: float32 [N] (device).
 * vals/meta come from sp24_compress with the same dtype, N and K.
 * Rules: M >= 0, N >= 0, N % 8 == 0 (N % 16 == 0 for SP24_OUT_INT8, so that
 * rows of Y stay 16-byte aligned); K >= 16, K % 16 == 0 (bf16) or
 * K % 32 == 0 (int8); alignment of 16 bytes for every pointer.  Ragged M, N
 * and K tails are handled in the kernel (no padding copies; [Orin ch.7] 6.2). */
sp24_status sp24_gemm(const void* X, int64_t M, int64_t K, const void* vals,
                      const void* meta, int64_t N, int dtype, const float* s_x,
                      const float* s_w, int out_kind, const float* s_y, void* Y,
                      void* stream);

/* The launch sp24_gemm makes for an M x N x K problem of `dtype` on the
 * current device (the pages fix no kernel design; this reports the one this
 * library chose, for profiling and tests).  Fills *plan; allocates nothing
 * and launches nothing.  The SP24_GEMM_IMPL environment variable, if set
 * (pair256, pair240, pair224, pair192, pair128, single, splitk), overrides
 * the kernel choice exactly as it does for sp24_gemm, and SP24_SPLITK (1..8)
 * the split-K kernel's split (tuning overrides; results never depend on
 * them beyond float32 summation order).
 *   kernel:        "splitk" (few tokens or tiles: K split across a cluster),
 *                  "single" (persistent, one 128 x 128 tile per SM at a time),
 *                  "pairNNN" (persistent, a CTA pair on two SMs computes
 *                  256-channel x NNN-token tiles with tcgen05 cta_group::2).
 *   tile_tokens, tile_channels: output tile (rows of Y x columns of Y).
 *   split_k:       K slices per tile (1 unless "splitk").
 *   ctas, cluster: CTAs launched and CTAs per cluster.
 * Errors: SP24_ERR_ARG for a NULL plan, M < 1, N < 1, K < 16 or an unknown
 * dtype; SP24_ERR_CUDA if the device cannot be queried. */
typedef struct sp24_gemm_plan_t {
  char kernel[16];
  int32_t tile_tokens;
  int32_t tile_channels;
  int32_t split_k;
  int32_t cluster;
  int64_t ctas;
} sp24_gemm_plan_t;

sp24_status sp24_gemm_plan(int64_t M, int64_t N, int64_t K, int dtype, sp24_gemm_plan_t* plan);

/* ------------------------------------------------------ 3x3 convolution */

/* 3x3 convolution input as the token operand of sp24_gemm ([Orin ch.7]
 * 2.2 A.3: large 3x3 convolutions at large batch or high resolution are good
 * 2:4 candidates; 2.1: groups of 4 run along the input channels).  Stride 1,
 * zero padding 1, NHWC:
 *   A[(b*H + h)*W + w][(kh*3 + kw)*C + c] = X[b][h+kh-1][w+kw-1][c], or 0
 *   when (h+kh-1, w+kw-1) lies outside the H x W image.
 * sp24_gemm(A, M = B*H*W, K = 9*C, ...) with the weights W[Cout][3][3][C]
 * pruned and compressed as the [Cout][9*C] matrix then gives the convolution
 * output Y[B*H*W][Cout] (NHWC); with C % 4 == 0 every group of 4 lies inside
 * one (kh, kw) tap.  For INT8, quantise X first (elem_bytes 1): a padded 0 is
 * the int8 code 0.
 *   X: [B][H][W][C] elements of elem_bytes bytes (2: bf16, 1: int8).
 *   A: [B*H*W][9*C] elements of the same size (written).
 * Rules: B, H, W, C >= 0; elem_bytes in {1, 2}; C * elem_bytes % 16 == 0. */
sp24_status sp24_im2col3x3(const void* X, int64_t B, int64_t H, int64_t W, int64_t C,
                           int elem_bytes, void* A, void* stream);

/* 3x3 convolution as an implicit sparse GEMM ([Orin ch.7] 2.2 A.3: large
 * 3x3 convolutions at large batch or high resolution are good 2:4
 * candidates; 2.1: groups of 4 run along the input channels).  Stride 1, zero
 * padding 1, NHWC:
 *   Y[(b*H + h)*W + w][co] = sum_{kh, kw, c} X[b][h+kh-1][w+kw-1][c] * W'[co][kh][kw][c]
 * with X zero outside the H x W image, i.e. sp24_gemm of the
 * sp24_im2col3x3 operand, computed without forming that operand: the GEMM's
 * token tiles are read straight from X (whole image rows per tile, the tap's
 * shift in the load coordinates, the padding from the loads' zero fill).
 *   X: [B][H][W][C] bf16 (dtype SP24_BF16) or int8 codes (SP24_INT8, from
 *      sp24_quantize; a padded 0 is the code 0).
 *   vals, meta: W[Cout][3][3][C] pruned and compressed as the [Cout][9*C]
 *      matrix (sp24_prune / sp24_compress with K = 9*C; with C % 4 == 0
 *      every group of 4 lies inside one tap).
 *   s_x, s_w, out_kind, s_y, Y: as sp24_gemm with M = B*H*W and N = Cout;
 *      Y is [B][H][W][Cout].
 * Rules: C * element bytes % 128 == 0 (C % 64 == 0 for bf16, C % 128 == 0
 * for int8), Cout % 8 == 0 (Cout % 16 == 0 for SP24_OUT_INT8), pointers
 * 16-byte aligned.  Image rows must tile the GEMM's token tiles: there must be
 * an r dividing H with (r * W) % 8 == 0 and r * W dividing 128 or 112 (e.g.
 * W = 8, 16, 32, 56, 64, 112 or 128 with r = 1, or W = 28 with even H);
 * otherwise the call returns SP24_ERR_UNSUPPORTED before any launch, and
 * sp24_im2col3x3 followed by sp24_gemm computes the same convolution.  Up to
 * 128 output channels run on single-SM tiles of 128 channels, more on CTA
 * pairs of 256 channels. */
sp24_status sp24_conv3x3(const void* X, int64_t B, int64_t H, int64_t W, int64_t C,
                         const void* vals, const void* meta, int64_t Cout, int dtype,
                         const float* s_x, const float* s_w, int out_kind, const float* s_y,
                         void* Y, void* stream);

/* ------------------------------------------------- allocation-free variant */

/* Largest K accepted by sp24_prune_wanda_noalloc. */
#define SP24_NOALLOC_MAX_K 65536

/* Wanda pruning for callers that cannot allocate device memory.  It computes
 * exactly what sp24_prune(W, N, K, Xc, Mc, SP24_WANDA, n_keep, mask_in,
 * mask_out, workspace, stream) computes, but keeps the float64 column norms in
 * a scratch array inside the library instead of a caller workspace, so the
 * caller passes only inputs and outputs.  Meant for code that must not call
 * cudaMalloc: inference engines and plugins whose device memory plan is fixed
 * at start-up, and code that runs where allocation would synchronise the
 * device or is not permitted.  (The pages have no counterpart; this is an
 * interface convenience.)
 *   - The scratch array holds SP24_NOALLOC_MAX_K doubles (512 KiB); every GPU
 *     that loads the library keeps it until the process exits.  K larger than
 *     SP24_NOALLOC_MAX_K returns SP24_ERR_UNSUPPORTED before any launch.
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up per device, repeated only if the device's context has
 *     changed since, e.g. after cudaDeviceReset); make that first call before
 *     any stream capture on the device.
 *   - All calls share the one array and each call overwrites all K entries it
 *     uses before reading them.  Calls that overlap on the GPU (for example on
 *     two streams at once) race on it and must be serialised by the caller.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Arguments, rules and errors are those of sp24_prune with mode SP24_WANDA. */
sp24_status sp24_prune_wanda_noalloc(const void* W, int64_t N, int64_t K, const void* Xc,
                                     int64_t Mc, int n_keep, const uint8_t* mask_in,
                                     uint8_t* mask_out, void* stream);

/* --------------------------------------------------------------- status */

/* Self-test of the failure path (the pages have no counterpart): launches one
 * thread that waits, with the same bounded mbarrier wait every kernel of the
 * library uses but a limit of limit_ns nanoseconds (1 .. 1e9), on a barrier
 * nothing arrives at.  The wait gives up, records SP24_ERR_TIMEOUT in the
 * device status word and the kernel returns normally: nothing traps or
 * hangs, and the context stays usable.  The next sp24_device_status() on the
 * stream reports (and clears) SP24_ERR_TIMEOUT.
 * Errors: SP24_ERR_ARG for a limit out of range. */
sp24_status sp24_selftest_wait_timeout(int64_t limit_ns, void* stream);

/* Synchronises `stream`, then returns and clears the device status word of the
 * current device (SP24_OK, SP24_ERR_PATTERN, SP24_ERR_TIMEOUT or SP24_ERR_INDEX), or
 * SP24_ERR_CUDA if the stream reports a CUDA error. */
sp24_status sp24_device_status(void* stream);

/* Static text for a status code (never NULL). */
const char* sp24_strerror(int status);

/* Text naming the last CUDA runtime / driver call that failed inside a libsp24
 * entry point on the calling thread and its error (e.g. "kernel launch:
 * cudaErrorInvalidValue"), or "" if none has failed.  Valid until the next
 * libsp24 call on this thread. */
const char* sp24_last_cuda_error(void);

/* Library version: major*10000 + minor*100 + patch. */
int sp24_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SP24_H_ */
