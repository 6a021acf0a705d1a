// libsp24: channel permutation search before masking, and the column gather
// that applies a permutation ([Orin ch.7] 3.1 workflow step 2 and 6.3: find
// an order of the input channels that gathers large weights into the same
// groups of 4 before the mask is made; permuting the same channels of X and W
// leaves Y = X W^T unchanged).
//
// Objective: the kept score, i.e. over every row and every group of 4 the sum
// of the n_keep largest scores.  Search: greedy pairwise exchange; each step
// exchanges the two channels (in different groups) whose exchange raises the
// kept score most, ties to the pair with the smallest lower index, then the
// smallest upper index; it stops when no exchange helps or after max_swaps.
// Every comparison is exact: the search runs on integer scores
// q = rint(s / s_max * 2^24) and accumulates in 64-bit integers.
//
// Algebra the kernels rely on.  For a group G and a member c, let R be the
// other three members' scores.  With k = n_keep,
//     keep(R + {v}) = base(c) + max(thr(c), v),
// base(c) = sum of the k-1 largest of R, thr(c) = the k-th largest of R.
// So exchanging a (group A) and b (group B) changes row r's kept score by
//     u_r(a) + u_r(b) + max(thr_r(a), q_r(b)) + max(thr_r(b), q_r(a)),
// u_r(c) = base_r(c) - keep_r(group of c), and the gain of the pair is
//     gain[a][b] = U(a) + U(b) + M[a][b] + M[b][a],
//     U(c) = sum_r u_r(c),   M[a][b] = sum_r max(thr_r(a), q_r(b)).
// An exchange only changes thr and u of the 8 members of the two groups, so
// after it only the rows and columns of gain for those 8 channels change.
//
// Device state (one workspace, sp24_permute_workspace_bytes):
//   q, thr   int32 [N][K]      integer scores, thr of the current grouping
//   tc       int32 [16][N]     thr (slots 0-7) and q (slots 8-15) of the 8
//                              channels of the last exchange, column-major
//   gain     int64 [K][K]      swap gains; NO_PAIR for same-group pairs
//   U        int64 [K]
//   part     int64 [2][8][K]   M[c][b] + M[b][c] for the 8 changed channels
//                              (two buffers, alternate steps)
//   best     int64 [K], int32 [K]  per row of gain: the largest entry and the
//                              smallest column holding it
//   pos      int32 [K]         inverse of perm
#include <algorithm>
#include <climits>

#include "sp24_device.cuh"
#include "sp24_host.h"

namespace sp24 {
namespace perm {

constexpr double kScale = 16777216.0;          // 2^24
constexpr long long kNoPair = LLONG_MIN;
constexpr int kGainTile = 64;                  // channels per side of a gain tile
constexpr int kRowChunk = 32;                  // rows per shared-memory stage

struct State {
  unsigned long long smax_bits;   // largest score, float64 bits (scores are >= 0)
  long long swaps;
  long long before;               // kept score of the identity order
  long long after;                // kept score of the current order
  int done;
  int ga, gb;                     // groups of the last exchange
  int pad;
};

struct Ws {
  State* st;
  int32_t* q;
  int32_t* thr;
  int32_t* tc;
  long long* gain;
  long long* u;
  long long* part;
  long long* best_val;
  int32_t* best_idx;
  int32_t* pos;
  int32_t* perm;
  int64_t n, k;
  int n_keep;
};

__device__ __forceinline__ void red_add(long long* p, long long v) {
  atomicAdd(reinterpret_cast<unsigned long long*>(p), static_cast<unsigned long long>(v));
}

// Score of one weight: |w| (magnitude) or |w| * norms[j] (Wanda), float64; a
// score that is not a finite positive number counts as 0.
__device__ __forceinline__ double weight_score(uint16_t bits, const double* norms, int64_t j) {
  const double a = fabs(static_cast<double>(__uint_as_float(static_cast<uint32_t>(bits) << 16)));
  const double s = norms ? a * norms[j] : a;
  return (s > 0.0 && s <= 1.7976931348623157e308) ? s : 0.0;
}

// thr and u of the four members of one group in one row (see the file head).
__device__ __forceinline__ void group_terms(const int v[4], int n_keep, int thr[4], int u[4],
                                            int& keep) {
  int base[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int o0 = v[(i + 1) & 3], o1 = v[(i + 2) & 3], o2 = v[(i + 3) & 3];
    const int hi = max(o0, o1), lo = min(o0, o1);
    const int r1 = max(hi, o2), m = min(hi, o2);
    const int r2 = max(lo, m), r3 = min(lo, m);
    base[i] = n_keep == 2 ? r1 : r1 + r2;
    thr[i] = n_keep == 2 ? r2 : r3;
  }
  keep = base[0] + max(thr[0], v[0]);
#pragma unroll
  for (int i = 0; i < 4; ++i) u[i] = base[i] - keep;
}

// (value, index) maximum over a warp; equal values go to the smaller index.
__device__ __forceinline__ void warp_argmax(long long& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const long long ov = __shfl_xor_sync(0xffffffffu, v, off);
    const int oi = __shfl_xor_sync(0xffffffffu, i, off);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

__device__ __forceinline__ long long warp_sum(long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// ------------------------------------------------------------ set-up passes
__global__ void __launch_bounds__(256) perm_smax(const uint16_t* __restrict__ w,
                                                 const double* __restrict__ norms, Ws ws) {
  pdl_launch_dependents();
  pdl_wait_prior();
  double m = 0.0;
  for (int64_t r = blockIdx.y; r < ws.n; r += gridDim.y)
    for (int64_t j = blockIdx.x * 256 + threadIdx.x; j < ws.k; j += gridDim.x * 256)
      m = fmax(m, weight_score(w[r * ws.k + j], norms, j));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0 && m > 0.0)
    atomicMax(&ws.st->smax_bits, static_cast<unsigned long long>(__double_as_longlong(m)));
}

__global__ void __launch_bounds__(256) perm_quantize(const uint16_t* __restrict__ w,
                                                     const double* __restrict__ norms, Ws ws) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const double smax = __longlong_as_double(static_cast<long long>(ws.st->smax_bits));
  for (int64_t r = blockIdx.y; r < ws.n; r += gridDim.y)
    for (int64_t j = blockIdx.x * 256 + threadIdx.x; j < ws.k; j += gridDim.x * 256) {
      int q = 0;
      if (smax > 0.0) q = static_cast<int>(rint(__ddiv_rn(weight_score(w[r * ws.k + j], norms, j),
                                                           smax) * kScale));
      ws.q[r * ws.k + j] = q;
    }
  if (blockIdx.y == 0)
    for (int64_t j = blockIdx.x * 256 + threadIdx.x; j < ws.k; j += gridDim.x * 256) {
      ws.perm[j] = static_cast<int32_t>(j);
      ws.pos[j] = static_cast<int32_t>(j);
    }
}

// thr and U of every group of the identity order, and the kept score.  One
// thread per group (groups are 4 consecutive channels), `rows` rows per
// block row.
__global__ void __launch_bounds__(256) perm_refresh_all(Ws ws, int64_t rows) {
  pdl_wait_prior();
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const bool live = g < ws.k / 4;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows;
  const int64_t r1 = min(ws.n, r0 + rows);
  long long uacc[4] = {0, 0, 0, 0};
  long long kacc = 0;
  if (live) {
    for (int64_t r = r0; r < r1; ++r) {
      const int4 qv = *reinterpret_cast<const int4*>(ws.q + r * ws.k + 4 * g);
      const int v[4] = {qv.x, qv.y, qv.z, qv.w};
      int t[4], u[4], keep;
      group_terms(v, ws.n_keep, t, u, keep);
      *reinterpret_cast<int4*>(ws.thr + r * ws.k + 4 * g) = make_int4(t[0], t[1], t[2], t[3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) uacc[i] += u[i];
      kacc += keep;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) red_add(ws.u + 4 * g + i, uacc[i]);
  }
  kacc = warp_sum(kacc);
  if ((threadIdx.x & 31) == 0 && kacc != 0) {
    red_add(&ws.st->before, kacc);
    red_add(&ws.st->after, kacc);
  }
  pdl_launch_dependents();
}

// M[a][b] + M[b][a] for every pair of channels, one 64 x 64 tile of pairs
// (upper triangle of tiles) per block over one slice of the rows.  gridDim.y
// > 1 splits the rows and adds into a zeroed gain; otherwise it stores.
__global__ void __launch_bounds__(256) perm_gain_full(Ws ws, int tiles, int64_t rows) {
  pdl_wait_prior();
  __shared__ int4 sm[4][kRowChunk][kGainTile / 4];   // thr_A, q_A, thr_B, q_B
  int64_t idx = blockIdx.x;
  int ti = 0;
  while (idx >= tiles - ti) {
    idx -= tiles - ti;
    ++ti;
  }
  const int tj = ti + static_cast<int>(idx);
  const int64_t a0 = static_cast<int64_t>(ti) * kGainTile, b0 = static_cast<int64_t>(tj) * kGainTile;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.y) * rows;
  const int64_t r_end = min(ws.n, r_begin + rows);
  long long acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0;
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kRowChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < 4 * kRowChunk * (kGainTile / 4); e += 256) {
      const int arr = e / (kRowChunk * (kGainTile / 4));
      const int rem = e % (kRowChunk * (kGainTile / 4));
      const int rr = rem / (kGainTile / 4), c4 = rem % (kGainTile / 4);
      const int64_t r = r0 + rr;
      const int64_t col = (arr < 2 ? a0 : b0) + 4 * c4;
      int4 v = make_int4(0, 0, 0, 0);   // rows past the slice add max(0, 0) = 0
      if (r < r_end && col < ws.k)
        v = *reinterpret_cast<const int4*>(((arr & 1) ? ws.q : ws.thr) + r * ws.k + col);
      sm[arr][rr][c4] = v;
    }
    __syncthreads();
    int a32[4][4];   // 32 rows x 2 terms x 2^24 stays below 2^31
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) a32[i][j] = 0;
#pragma unroll 4
    for (int rr = 0; rr < kRowChunk; ++rr) {
      const int4 ta = sm[0][rr][ty], qa = sm[1][rr][ty], tb = sm[2][rr][tx], qb = sm[3][rr][tx];
      const int tav[4] = {ta.x, ta.y, ta.z, ta.w}, qav[4] = {qa.x, qa.y, qa.z, qa.w};
      const int tbv[4] = {tb.x, tb.y, tb.z, tb.w}, qbv[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) a32[i][j] += max(tav[i], qbv[j]) + max(tbv[j], qav[i]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += a32[i][j];
  }
  const bool split = gridDim.y > 1;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t a = a0 + 4 * ty + i;
    if (a >= ws.k) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t b = b0 + 4 * tx + j;
      if (b >= ws.k) continue;
      long long* ab = ws.gain + a * ws.k + b;
      long long* ba = ws.gain + b * ws.k + a;
      if (split) {
        red_add(ab, acc[i][j]);
        if (ti != tj) red_add(ba, acc[i][j]);
      } else {
        *ab = acc[i][j];
        if (ti != tj) *ba = acc[i][j];
      }
    }
  }
  pdl_launch_dependents();
}

// Finishes gain (adds U, marks same-group pairs) and the best entry of every
// row.  One warp per row.
__global__ void __launch_bounds__(256) perm_rowbest_full(Ws ws) {
  pdl_wait_prior();
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t a = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); a < ws.k; a += warps) {
    const int ga = ws.pos[a] >> 2;
    const long long ua = ws.u[a];
    long long bv = kNoPair;
    int bi = INT_MAX;
    for (int64_t b = lane; b < ws.k; b += 32) {
      long long v = kNoPair;
      if ((ws.pos[b] >> 2) != ga) v = ws.gain[a * ws.k + b] + ua + ws.u[b];
      ws.gain[a * ws.k + b] = v;
      if (v > bv) {
        bv = v;
        bi = static_cast<int>(b);
      }
    }
    warp_argmax(bv, bi);
    if (lane == 0) {
      ws.best_val[a] = bv;
      ws.best_idx[a] = bi;
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------- one greedy step
// The kernels of a step (and the longer set-up passes) signal their
// dependents only after their main work: an early signal would let the next
// kernel's blocks occupy SM slots while they wait.  `part` is double-buffered by the parity of the exchange
// count: step t accumulates into part[t & 1] and, while reading it, clears
// part[(t + 1) & 1], which step t + 1 accumulates into.

// (1) Picks the best pair from the row bests, exchanges it in perm / pos and
// clears U of the 8 channels of the two groups.  One block.
__global__ void __launch_bounds__(1024) perm_pick(Ws ws, int64_t max_swaps) {
  pdl_wait_prior();
  State* st = ws.st;
  if (st->done) return;
  const long long swaps_now = st->swaps;   // read by every thread before thread 0 writes it
  __shared__ long long s_val[32];
  __shared__ int s_idx[32];
  __shared__ int s_g[2];
  long long bv = kNoPair;
  int ba = INT_MAX;
  for (int64_t a = threadIdx.x; a < ws.k; a += 1024) {
    const long long v = ws.best_val[a];
    if (v > bv) {
      bv = v;
      ba = static_cast<int>(a);
    }
  }
  warp_argmax(bv, ba);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_val[warp] = bv;
    s_idx[warp] = ba;
  }
  __syncthreads();
  bv = s_val[lane];
  ba = s_idx[lane];
  warp_argmax(bv, ba);   // every warp now holds the block result
  if (bv <= 0 || swaps_now >= max_swaps) {
    if (threadIdx.x == 0) st->done = 1;
    return;
  }
  if (threadIdx.x == 0) {
    const int b = ws.best_idx[ba];
    const int pa = ws.pos[ba], pb = ws.pos[b];
    ws.perm[pa] = b;
    ws.perm[pb] = ba;
    ws.pos[ba] = pb;
    ws.pos[b] = pa;
    st->ga = pa >> 2;
    st->gb = pb >> 2;
    st->swaps = swaps_now + 1;
    st->after += bv;
    s_g[0] = pa >> 2;
    s_g[1] = pb >> 2;
  }
  __syncthreads();
  if (threadIdx.x < 8) ws.u[ws.perm[4 * s_g[threadIdx.x >> 2] + (threadIdx.x & 3)]] = 0;
  pdl_launch_dependents();
}

// (2) thr and U of the two exchanged groups; also the column-major copies of
// their thr and q for step (3).  One thread per row, blockIdx.y = group.
__global__ void __launch_bounds__(256) perm_refresh_pair(Ws ws) {
  pdl_wait_prior();
  if (ws.st->done) return;
  const int slot0 = 4 * blockIdx.y;
  const int g = blockIdx.y == 0 ? ws.st->ga : ws.st->gb;
  int c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) c[i] = ws.perm[4 * g + i];
  long long uacc[4] = {0, 0, 0, 0};
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; r < ws.n;
       r += static_cast<int64_t>(gridDim.x) * 256) {
    int v[4], t[4], u[4], keep;
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = ws.q[r * ws.k + c[i]];
    group_terms(v, ws.n_keep, t, u, keep);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ws.thr[r * ws.k + c[i]] = t[i];
      ws.tc[(slot0 + i) * ws.n + r] = t[i];
      ws.tc[(8 + slot0 + i) * ws.n + r] = v[i];
      uacc[i] += u[i];
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long s = warp_sum(uacc[i]);
    if ((threadIdx.x & 31) == 0 && s != 0) red_add(ws.u + c[i], s);
  }
  pdl_launch_dependents();
}

// (3) part[i][b] = M[c_i][b] + M[b][c_i] for the 8 changed channels c_i and
// every channel b: one thread per b over one slice of the rows.  Eight rows
// of q and thr are loaded before they are used, to keep loads in flight.
__global__ void __launch_bounds__(256) perm_partial(Ws ws, int64_t rows) {
  pdl_wait_prior();
  if (ws.st->done) return;
  long long* part = ws.part + (ws.st->swaps & 1) * 8 * ws.k;
  __shared__ int4 stc[kRowChunk][4];   // per row: thr of slots 0-7, q of slots 0-7
  const int64_t b = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  const bool live = b < ws.k;
  const int64_t r_begin = static_cast<int64_t>(blockIdx.y) * rows;
  const int64_t r_end = min(ws.n, r_begin + rows);
  long long acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t r0 = r_begin; r0 < r_end; r0 += kRowChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * kRowChunk; e += 256) {
      const int slot = e / kRowChunk, rr = e % kRowChunk;
      const int64_t r = r0 + rr;
      reinterpret_cast<int*>(&stc[rr][0])[slot] = r < r_end ? ws.tc[slot * ws.n + r] : 0;
    }
    __syncthreads();
    const int cnt = static_cast<int>(min(static_cast<int64_t>(kRowChunk), r_end - r0));
    int a32[8] = {0, 0, 0, 0, 0, 0, 0, 0};   // 32 rows x 2 terms x 2^24 < 2^31
    if (live) {
      for (int rb = 0; rb < cnt; rb += 8) {
        int qb[8], tb[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const bool in = rb + j < cnt;
          const int64_t off = (r0 + rb + (in ? j : 0)) * ws.k + b;
          qb[j] = in ? __ldg(ws.q + off) : 0;
          tb[j] = in ? __ldg(ws.thr + off) : 0;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (rb + j >= cnt) break;
          const int4 t0 = stc[rb + j][0], t1 = stc[rb + j][1];
          const int4 q0 = stc[rb + j][2], q1 = stc[rb + j][3];
          const int tcv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
          const int qcv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) a32[i] += max(tcv[i], qb[j]) + max(tb[j], qcv[i]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += a32[i];
  }
  if (live) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red_add(part + i * ws.k + b, acc[i]);
  }
  pdl_launch_dependents();
}

// (4) New gain rows / columns of the 8 changed channels and the row bests.
// A row outside the two groups only needs a full rescan when its old best
// partner is one of the 8; otherwise its other entries did not change.  Also
// clears the other part buffer for the next step.
__global__ void __launch_bounds__(256) perm_update(Ws ws) {
  pdl_wait_prior();
  if (ws.st->done) return;
  const int ga = ws.st->ga, gb = ws.st->gb;
  const long long par = ws.st->swaps & 1;
  const long long* part = ws.part + par * 8 * ws.k;
  long long* next = ws.part + (par ^ 1) * 8 * ws.k;
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; e < 8 * ws.k;
       e += static_cast<int64_t>(gridDim.x) * 256)
    next[e] = 0;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * 8;
  for (int64_t a = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5); a < ws.k; a += warps) {
    const int pa = ws.pos[a];
    const int grp = pa >> 2;
    const long long ua = ws.u[a];
    long long* row = ws.gain + a * ws.k;
    long long bv = kNoPair;
    int bi = INT_MAX;
    if (grp == ga || grp == gb) {
      const int slot = (grp == ga ? 0 : 4) + (pa & 3);
      for (int64_t b = lane; b < ws.k; b += 32) {
        long long v = kNoPair;
        if ((ws.pos[b] >> 2) != grp) v = ua + ws.u[b] + part[slot * ws.k + b];
        row[b] = v;
        if (v > bv) {
          bv = v;
          bi = static_cast<int>(b);
        }
      }
    } else {
      if (lane < 8) {
        const int c = ws.perm[4 * (lane < 4 ? ga : gb) + (lane & 3)];
        const long long v = ua + ws.u[c] + part[lane * ws.k + a];
        row[c] = v;
        bv = v;
        bi = c;
      }
      const int old = ws.best_idx[a];
      const int og = (old >= 0 && old < ws.k) ? (ws.pos[old] >> 2) : -1;
      if (og != ga && og != gb) {
        if (lane == 0) {
          const long long ov = ws.best_val[a];
          if (ov > bv || (ov == bv && old < bi)) {
            bv = ov;
            bi = old;
          }
        }
      } else {
        // the 8 new entries are in `row` now; scan it two entries at a time
        __syncwarp();
        const longlong2* row2 = reinterpret_cast<const longlong2*>(row);
        for (int64_t h = lane; h < ws.k / 2; h += 32) {
          const longlong2 v = row2[h];
          if (v.x > bv || (v.x == bv && static_cast<int>(2 * h) < bi)) {
            bv = v.x;
            bi = static_cast<int>(2 * h);
          }
          if (v.y > bv || (v.y == bv && static_cast<int>(2 * h + 1) < bi)) {
            bv = v.y;
            bi = static_cast<int>(2 * h + 1);
          }
        }
      }
    }
    warp_argmax(bv, bi);
    if (lane == 0) {
      ws.best_val[a] = bv;
      ws.best_idx[a] = bi;
    }
  }
  pdl_launch_dependents();
}

// ------------------------------------------------------------- column gather
template <class T>
__global__ void __launch_bounds__(256) gather_columns(const T* __restrict__ in, int64_t rows,
                                                      int64_t k, const int32_t* __restrict__ perm,
                                                      T* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait_prior();
  for (int64_t j = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; j < k;
       j += static_cast<int64_t>(gridDim.x) * 256) {
    const int32_t p = perm[j];
    const bool ok = p >= 0 && p < k;
    if (!ok && blockIdx.y == 0) raise_error(kErrIndexBit);
    for (int64_t r = blockIdx.y; r < rows; r += gridDim.y)
      out[r * k + j] = ok ? in[r * k + p] : T(0);
  }
}

// Workspace carving, 256-byte aligned pieces.
struct Layout {
  size_t st, q, thr, tc, gain, u, part, best_val, best_idx, pos, total;
};

inline size_t up256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

inline Layout layout(int64_t n, int64_t k) {
  Layout l;
  size_t o = 0;
  const size_t nk = static_cast<size_t>(n) * static_cast<size_t>(k);
  l.st = o;        o += up256(sizeof(State));
  l.q = o;         o += up256(4 * nk);
  l.thr = o;       o += up256(4 * nk);
  l.tc = o;        o += up256(4 * 16 * static_cast<size_t>(n));
  l.gain = o;      o += up256(8 * static_cast<size_t>(k) * static_cast<size_t>(k));
  l.u = o;         o += up256(8 * static_cast<size_t>(k));
  l.part = o;      o += up256(2 * 8 * 8 * static_cast<size_t>(k));
  l.best_val = o;  o += up256(8 * static_cast<size_t>(k));
  l.best_idx = o;  o += up256(4 * static_cast<size_t>(k));
  l.pos = o;       o += up256(4 * static_cast<size_t>(k));
  l.total = o;
  return l;
}

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Rows per slice so that `blocks` x slices covers about `waves` waves, slices of
// at least `min_rows` rows, a multiple of kRowChunk.
inline int64_t slice_rows(int64_t n, int64_t blocks, int64_t min_rows, int waves = 2) {
  const int64_t want = waves * static_cast<int64_t>(sm_count());
  int64_t slices = blocks >= want ? 1 : ceil_div(want, blocks);
  slices = std::min(slices, std::max<int64_t>(1, ceil_div(n, min_rows)));
  const int64_t rows = ceil_div(ceil_div(n, slices), kRowChunk) * kRowChunk;
  return rows;
}

}  // namespace perm
}  // namespace sp24

using namespace sp24;

extern "C" {

size_t sp24_permute_workspace_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 4 || K % 4 != 0 || K > SP24_PERMUTE_MAX_K) return 0;
  return perm::layout(N, K).total;
}

sp24_status sp24_permute_search(const void* W, int64_t N, int64_t K, const double* norms,
                                int n_keep, int64_t max_swaps, int32_t* perm_out,
                                void* workspace, size_t workspace_bytes,
                                sp24_permute_result_t* result, void* stream) {
  using namespace perm;
  if (!W || !perm_out || !workspace || N < 1 || K < 4 || max_swaps < 0) return SP24_ERR_ARG;
  if (n_keep != 2 && n_keep != 3) return SP24_ERR_ARG;
  if (K % 4 != 0 || K > SP24_PERMUTE_MAX_K) return SP24_ERR_ALIGN;
  if (!aligned16(W) || !aligned16(perm_out) || !aligned16(workspace) ||
      (norms && !aligned16(norms)))
    return SP24_ERR_ALIGN;
  const Layout l = layout(N, K);
  if (workspace_bytes < l.total) return SP24_ERR_ARG;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  char* base = static_cast<char*>(workspace);
  Ws ws;
  ws.st = reinterpret_cast<State*>(base + l.st);
  ws.q = reinterpret_cast<int32_t*>(base + l.q);
  ws.thr = reinterpret_cast<int32_t*>(base + l.thr);
  ws.tc = reinterpret_cast<int32_t*>(base + l.tc);
  ws.gain = reinterpret_cast<long long*>(base + l.gain);
  ws.u = reinterpret_cast<long long*>(base + l.u);
  ws.part = reinterpret_cast<long long*>(base + l.part);
  ws.best_val = reinterpret_cast<long long*>(base + l.best_val);
  ws.best_idx = reinterpret_cast<int32_t*>(base + l.best_idx);
  ws.pos = reinterpret_cast<int32_t*>(base + l.pos);
  ws.perm = perm_out;
  ws.n = N;
  ws.k = K;
  ws.n_keep = n_keep;
  const uint16_t* w = static_cast<const uint16_t*>(W);

  cudaError_t e = cudaMemsetAsync(ws.st, 0, sizeof(State), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.u, 0, 8 * static_cast<size_t>(K), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws.part, 0, 2 * 8 * 8 * static_cast<size_t>(K), s);
  if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync", e);

  const unsigned ex = static_cast<unsigned>(std::min<int64_t>(ceil_div(K, 256), 8));
  const unsigned ey = static_cast<unsigned>(std::min<int64_t>(N, std::max<int64_t>(1, 2048 / ex)));
  SP24_TRY(launch_kernel(perm_smax, dim3(ex, ey), dim3(256), 0, s, 1, w, norms, ws));
  SP24_TRY(launch_kernel(perm_quantize, dim3(ex, ey), dim3(256), 0, s, 1, w, norms, ws));

  const int64_t groups = K / 4;
  const int64_t gx = ceil_div(groups, 256);
  const int64_t rrows = std::max<int64_t>(64, slice_rows(N, gx, 64));
  SP24_TRY(launch_kernel(perm_refresh_all, dim3(static_cast<unsigned>(gx),
                                                static_cast<unsigned>(ceil_div(N, rrows))),
                         dim3(256), 0, s, 1, ws, rrows));

  const int tiles = static_cast<int>(ceil_div(K, kGainTile));
  const int64_t ntiles = static_cast<int64_t>(tiles) * (tiles + 1) / 2;
  const int64_t grows = slice_rows(N, ntiles, 128);
  const int64_t gsplit = ceil_div(N, grows);
  if (gsplit > 1) {
    e = cudaMemsetAsync(ws.gain, 0, 8 * static_cast<size_t>(K) * static_cast<size_t>(K), s);
    if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync", e);
  }
  SP24_TRY(launch_kernel(perm_gain_full, dim3(static_cast<unsigned>(ntiles),
                                              static_cast<unsigned>(gsplit)),
                         dim3(256), 0, s, 1, ws, tiles, grows));
  const unsigned wrows = static_cast<unsigned>(std::min<int64_t>(ceil_div(K, 8), 4096));
  SP24_TRY(launch_kernel(perm_rowbest_full, dim3(wrows), dim3(256), 0, s, 1, ws));

  const int64_t pcols = ceil_div(K, 256);
  const int64_t prows = slice_rows(N, pcols, 64, 4);
  const dim3 pgrid(static_cast<unsigned>(pcols), static_cast<unsigned>(ceil_div(N, prows)));
  const unsigned fx = static_cast<unsigned>(std::min<int64_t>(ceil_div(N, 256), 64));
  if (max_swaps > (INT64_MAX >> 1)) max_swaps = INT64_MAX >> 1;
  State host{};
  int64_t launched = 0;
  int64_t batch = 16;
  // Each step makes at most one exchange and the step after the last one
  // sets `done`; max_swaps + 1 steps always reach it.
  while (launched <= max_swaps) {
    const int64_t steps = std::min(batch, max_swaps + 1 - launched);
    for (int64_t i = 0; i < steps; ++i) {
      SP24_TRY(launch_kernel(perm_pick, dim3(1), dim3(1024), 0, s, 1, ws, max_swaps));
      SP24_TRY(launch_kernel(perm_refresh_pair, dim3(fx, 2), dim3(256), 0, s, 1, ws));
      SP24_TRY(launch_kernel(perm_partial, pgrid, dim3(256), 0, s, 1, ws, prows));
      SP24_TRY(launch_kernel(perm_update, dim3(wrows), dim3(256), 0, s, 1, ws));
    }
    launched += steps;
    e = cudaMemcpyAsync(&host, ws.st, sizeof(State), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail("search status copy", e);
    if (host.done) break;
    batch = std::min<int64_t>(batch * 2, 512);
  }
  if (!host.done) return SP24_ERR_TIMEOUT;   // unreachable: max_swaps + 1 steps ran
  if (result) {
    result->swaps = host.swaps;
    result->kept_before = host.before;
    result->kept_after = host.after;
  }
  return SP24_OK;
}

sp24_status sp24_permute_columns(const void* A, int64_t rows, int64_t K, int elem_bytes,
                                 const int32_t* perm, void* A_out, void* stream) {
  if (rows < 0 || K < 0) return SP24_ERR_ARG;
  if (elem_bytes != 1 && elem_bytes != 2 && elem_bytes != 4) return SP24_ERR_ARG;
  if (rows == 0 || K == 0) return SP24_OK;
  if (!A || !perm || !A_out || A == A_out) return SP24_ERR_ARG;
  if (K > INT32_MAX) return SP24_ERR_ARG;
  if (!aligned16(A) || !aligned16(perm) || !aligned16(A_out)) return SP24_ERR_ALIGN;
  SP24_TRY(check_device());
  cudaStream_t s = as_stream(stream);
  const unsigned gx = static_cast<unsigned>(std::min<int64_t>(perm::ceil_div(K, 256), 64));
  const unsigned gy = static_cast<unsigned>(std::min<int64_t>(rows, std::max<int64_t>(1, 4096 / gx)));
  if (elem_bytes == 1)
    return launch_kernel(perm::gather_columns<uint8_t>, dim3(gx, gy), dim3(256), 0, s, 1,
                         static_cast<const uint8_t*>(A), rows, K, perm,
                         static_cast<uint8_t*>(A_out));
  if (elem_bytes == 2)
    return launch_kernel(perm::gather_columns<uint16_t>, dim3(gx, gy), dim3(256), 0, s, 1,
                         static_cast<const uint16_t*>(A), rows, K, perm,
                         static_cast<uint16_t*>(A_out));
  return launch_kernel(perm::gather_columns<uint32_t>, dim3(gx, gy), dim3(256), 0, s, 1,
                       static_cast<const uint32_t*>(A), rows, K, perm,
                       static_cast<uint32_t*>(A_out));
}

}  // extern "C"
