"""CPU oracle for N:4 structured sparsity: pruning, compression, sparse GEMM.

TEST INFRASTRUCTURE ONLY.  Nothing in the library path imports, calls or
executes this module; only the tests, the package smoke check and the
benchmark's CPU-baseline leg do.  It shares no code, tables or constants with
the CUDA kernels.

Everything here is the plain definition written out in float64 / int64 with
numpy (a matmul, a sort/partition and an elementwise sqrt are the only library
primitives), so that it can be checked against the pages by eye.  The sources
("pages") are cited by title and section:

* [Ampere-sparsity] NVIDIA x Tencent MLPD article on Ampere fine-grained
  structured sparsity (nvidia.zhidx.com): the 2:4 pattern and its compressed
  format (Figure 1 and the paragraphs around it), progressive sparsity
  (Figures 3/4), quantisation "PTQ and QAT" (scale covering 99.99 %).
* [Wanda-2:4] "Structured Pruning: 2:4 sparse inference with the Wanda
  algorithm" (zyxy.net), section 1.3 (2:4 definition) and section 2.1/2.2
  (Wanda score |w_i| * sqrt(sum A_j^2), sort, prune the lowest).
* [Sparse-accel forum] oeforum.com post on sparse acceleration: 2-bit
  metadata per nonzero, the hardware fetches the matching activations.
* [Orin ch.7] "Chapter 7: 2:4 Structured Sparsity" (Orin NN design book),
  section 2.1 (groups of 4 along the input-channel K dimension; worked 1x4
  example: prune, compress to values + 2-bit indices, multiply with the
  selected activations), section 5 exercise Q1, section 6.1 (check every
  1x4 block before export).

Readings taken where the pages are silent or contradict one another:

* Exactly ``n_keep`` positions are kept per group of 4 (a kept value may itself
  be zero, so "at least two zeros" still holds for the values).
* Keep the largest scores; ties go to the lower index.  The worked figure in
  [Orin ch.7] 2.1 states this rule but draws a mask that does not follow it;
  the rule is followed, not the drawing.
* Groups are 4 consecutive entries along K within one row of W[N, K].
* Wanda activation statistic: the L2 norm over calibration tokens of input
  feature j, accumulated in float64 sequentially over the tokens.
* Progressive 25 % -> 50 %: the second mask is recomputed on W * mask1
  (dropped entries score 0).
* Metadata: ascending 2-bit positions; nibble = lo | hi << 2; group 2b sits in
  the low nibble of byte b.  Mask bytes use the same nibble placement with
  bit p set when position p is kept.
* INT8: symmetric, no zero point, q in [-127, 127], round half to even.  The
  scale is the nearest-rank ``coverage`` quantile of |v| divided by 127; a
  zero quantile gives scale 1.  Dequantisation is done in float32 in the order
  c = s_x * s_w[n]; f = float(acc); y = bf16_rne(f * c).
* Channel permutation search ([Orin ch.7] 3.1 and 6.3 give only the goal):
  the objective, the greedy exchange rule and the integer scores it compares
  are stated at that section below.

Parity pins for every function here are in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from typing import Optional, Tuple

import numpy as np

MAGNITUDE = "magnitude"
WANDA = "wanda"


# ---------------------------------------------------------------------------
# a1  Wanda column norms       [Wanda-2:4] section 2.1
# ---------------------------------------------------------------------------
def column_norms(xc: np.ndarray) -> np.ndarray:
    """n_j = sqrt(sum_t x_tj^2) over the calibration tokens t.

    ``xc`` is [Mc, K] float64 holding bf16 values exactly.  The sum runs in
    float64, one rounding per addition, sequentially in t = 0 .. Mc-1; the
    squares of bf16 values are exact in float64.
    """
    xc = np.asarray(xc, dtype=np.float64)
    acc = np.zeros(xc.shape[1], dtype=np.float64)
    for t in range(xc.shape[0]):
        acc = acc + xc[t] * xc[t]
    return np.sqrt(acc)


# ---------------------------------------------------------------------------
# a2  scores                    [Orin ch.7] 2.1, [Wanda-2:4] 2.1
# ---------------------------------------------------------------------------
def scores(w: np.ndarray, mode: str, norms: Optional[np.ndarray] = None) -> np.ndarray:
    """Magnitude: s = |w|.  Wanda: s = |w| * n_j (one float64 rounding)."""
    a = np.abs(np.asarray(w, dtype=np.float64))
    if mode == MAGNITUDE:
        return a
    if mode == WANDA:
        if norms is None:
            raise ValueError("wanda scoring needs column norms")
        return a * np.asarray(norms, dtype=np.float64)[None, :]
    raise ValueError(f"unknown mode {mode!r}")


# ---------------------------------------------------------------------------
# a3  top-n_keep of each group of 4 along K
#     [Ampere-sparsity] Figure 1, [Wanda-2:4] 1.3 and 2.2, [Orin ch.7] 2.1
# ---------------------------------------------------------------------------
def select(s: np.ndarray, n_keep: int) -> np.ndarray:
    """Boolean keep mask [N, K].

    Within each group of 4 consecutive scores along K, position p is kept iff
    fewer than ``n_keep`` other positions q beat it, where q beats p when
    s_q > s_p, or s_q == s_p and q < p (ties go to the lower index).
    """
    if n_keep not in (2, 3):
        raise ValueError("n_keep must be 2 or 3")
    s = np.asarray(s, dtype=np.float64)
    n, k = s.shape
    if k % 4:
        raise ValueError("K must be a multiple of 4")
    g = s.reshape(n, k // 4, 4)
    keep = np.zeros(g.shape, dtype=bool)
    for p in range(4):
        beaten_by = np.zeros(g.shape[:2], dtype=np.int64)
        for q in range(4):
            if q == p:
                continue
            beats = g[..., q] > g[..., p]
            if q < p:
                beats = beats | (g[..., q] == g[..., p])
            beaten_by += beats
        keep[..., p] = beaten_by < n_keep
    return keep.reshape(n, k)


def prune(w: np.ndarray, mode: str, n_keep: int, xc: Optional[np.ndarray] = None,
          mask_in: Optional[np.ndarray] = None) -> np.ndarray:
    """Keep mask of W (optionally of W * mask_in, the progressive second step).

    [Ampere-sparsity] progressive sparsity (Figure 4): mask to 25 % first,
    then recompute the mask on the remaining weights to reach 50 %.
    """
    w = np.asarray(w, dtype=np.float64)
    if mask_in is not None:
        w = np.where(np.asarray(mask_in, dtype=bool), w, 0.0)
    norms = column_norms(xc) if mode == WANDA else None
    return select(scores(w, mode, norms), n_keep)


def progressive(w: np.ndarray, mode: str, xc: Optional[np.ndarray] = None
                ) -> Tuple[np.ndarray, np.ndarray]:
    """mask1 = keep 3 of 4; mask2 = keep 2 of 4 on W * mask1."""
    m1 = prune(w, mode, 3, xc)
    m2 = prune(w, mode, 2, xc, mask_in=m1)
    return m1, m2


def pack_mask(keep: np.ndarray) -> np.ndarray:
    """[N, K] bool -> uint8 [N, K/8]: nibble per group, bit p = position p
    kept, group 2b in the low nibble of byte b."""
    keep = np.asarray(keep, dtype=bool)
    n, k = keep.shape
    if k % 8:
        raise ValueError("K must be a multiple of 8")
    g = keep.reshape(n, k // 4, 4).astype(np.uint8)
    nib = g[..., 0] | (g[..., 1] << 1) | (g[..., 2] << 2) | (g[..., 3] << 3)
    return (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)


def unpack_mask(packed: np.ndarray, k: int) -> np.ndarray:
    """Inverse of :func:`pack_mask`."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    nib = np.empty((n, k // 4), dtype=np.uint8)
    nib[:, 0::2] = packed & 0xF
    nib[:, 1::2] = packed >> 4
    bits = np.stack([(nib >> p) & 1 for p in range(4)], axis=-1)
    return bits.reshape(n, k).astype(bool)


# ---------------------------------------------------------------------------
# a4  compression to values + 2-bit metadata
#     [Ampere-sparsity] Figure 1; [Sparse-accel forum]; [Orin ch.7] 2.1 step 2
# ---------------------------------------------------------------------------
class PatternError(ValueError):
    """A group of 4 does not keep exactly two positions ([Orin ch.7] 6.1)."""


def compress(w: np.ndarray, keep: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Return (vals [N, K/2], meta uint8 [N, K/8]).

    vals[n, 2g] = w[n, 4g + lo], vals[n, 2g+1] = w[n, 4g + hi] with lo < hi
    the two kept positions of group g; the group's metadata nibble is
    lo | hi << 2 and group 2b sits in the low nibble of meta byte b.
    ``vals`` keeps the dtype of ``w``.
    """
    w = np.asarray(w)
    keep = np.asarray(keep, dtype=bool)
    n, k = w.shape
    if k % 8:
        raise ValueError("K must be a multiple of 8")
    kg = keep.reshape(n, k // 4, 4)
    if np.any(kg.sum(axis=-1) != 2):
        raise PatternError("every group of 4 must keep exactly 2 positions")
    wg = w.reshape(n, k // 4, 4)
    pos = np.argsort(~kg, axis=-1, kind="stable")[..., :2]   # kept positions, ascending
    lo, hi = pos[..., 0], pos[..., 1]
    vals = np.empty((n, k // 4, 2), dtype=w.dtype)
    vals[..., 0] = np.take_along_axis(wg, lo[..., None], axis=-1)[..., 0]
    vals[..., 1] = np.take_along_axis(wg, hi[..., None], axis=-1)[..., 0]
    nib = (lo | (hi << 2)).astype(np.uint8)
    meta = (nib[:, 0::2] | (nib[:, 1::2] << 4)).astype(np.uint8)
    return vals.reshape(n, k // 2), meta


def decompress(vals: np.ndarray, meta: np.ndarray, k: int) -> np.ndarray:
    """Dense W' [N, K] with the kept values at their positions, zeros elsewhere."""
    vals = np.asarray(vals)
    meta = np.asarray(meta, dtype=np.uint8)
    n = vals.shape[0]
    nib = np.empty((n, k // 4), dtype=np.uint8)
    nib[:, 0::2] = meta & 0xF
    nib[:, 1::2] = meta >> 4
    lo = (nib & 3).astype(np.int64)
    hi = (nib >> 2).astype(np.int64)
    out = np.zeros((n, k // 4, 4), dtype=vals.dtype)
    v = vals.reshape(n, k // 4, 2)
    np.put_along_axis(out, lo[..., None], v[..., 0:1], axis=-1)
    np.put_along_axis(out, hi[..., None], v[..., 1:2], axis=-1)
    return out.reshape(n, k)


# ---------------------------------------------------------------------------
# a6  sparse GEMM, floating point     [Orin ch.7] 2.1 step 3
# ---------------------------------------------------------------------------
def gemm(x: np.ndarray, vals: np.ndarray, meta: np.ndarray, k: int
         ) -> Tuple[np.ndarray, np.ndarray]:
    """Y = X * W'^T in float64 plus the per-element error scale
    a_mn = sum_k |x_mk * W'_nk| used by the bf16 tolerance."""
    x = np.asarray(x, dtype=np.float64)
    wd = decompress(np.asarray(vals, dtype=np.float64), meta, k)
    return x @ wd.T, np.abs(x) @ np.abs(wd).T


# ---------------------------------------------------------------------------
# a5  INT8 calibration and quantisation   [Ampere-sparsity] "PTQ and QAT"
# ---------------------------------------------------------------------------
def nearest_rank(coverage: float, count: int) -> int:
    """1-based nearest rank ceil(coverage * count), computed in IEEE double."""
    return max(1, int(math.ceil(coverage * count)))


def quantile_abs(v: np.ndarray, coverage: float) -> float:
    """Nearest-rank ``coverage`` quantile of |v| (the smallest |v| such that at
    least ``coverage`` of the values are <= it)."""
    a = np.abs(np.asarray(v, dtype=np.float64).ravel())
    if a.size == 0:
        return 0.0
    r = nearest_rank(coverage, a.size)
    return float(np.partition(a, r - 1)[r - 1])


def scale_from_quantile(t: float) -> np.float32:
    """s = float32(t) / 127 in float32; a zero quantile gives s = 1."""
    if t == 0.0:
        return np.float32(1.0)
    return np.float32(np.float32(t) / np.float32(127.0))


def channel_scales(w: np.ndarray, keep: np.ndarray, coverage: float = 0.9999) -> np.ndarray:
    """Per-output-channel weight scale over the kept entries of each row."""
    w = np.asarray(w, dtype=np.float64)
    keep = np.asarray(keep, dtype=bool)
    out = np.empty(w.shape[0], dtype=np.float32)
    for n in range(w.shape[0]):
        out[n] = scale_from_quantile(quantile_abs(w[n][keep[n]], coverage))
    return out


def tensor_scale(x: np.ndarray, coverage: float = 0.9999) -> np.float32:
    """Per-tensor activation scale over all entries of X."""
    return scale_from_quantile(quantile_abs(x, coverage))


def quantize(v: np.ndarray, s) -> np.ndarray:
    """q = clamp(rint(float32(v) / s), -127, 127), float32 IEEE divide,
    round half to even.  ``s`` is a scalar or broadcasts against ``v``."""
    q = np.rint(np.asarray(v, dtype=np.float32) / np.asarray(s, dtype=np.float32))
    return np.clip(q, -127, 127).astype(np.int8)


def bf16_rne(f: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even; returns the uint16 bit patterns.

    Keeps the top 16 bits of the float32 pattern, rounding on the dropped 16
    bits: add 0x7FFF plus the lowest kept bit, then truncate.  Finite inputs.
    """
    f = np.ascontiguousarray(np.asarray(f, dtype=np.float32))
    if not np.all(np.isfinite(f)):
        raise ValueError("bf16_rne expects finite inputs")
    b = f.view(np.uint32).astype(np.uint64)
    b = b + 0x7FFF + ((b >> 16) & 1)
    return (b >> 16).astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns as float64."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# a7  sparse GEMM, INT8 with int32 accumulation and dequantisation
#     [Sparse-accel forum] INT8 + 2:4; [Ampere-sparsity] "PTQ and QAT"
# ---------------------------------------------------------------------------
INT32_MIN, INT32_MAX = -(2 ** 31), 2 ** 31 - 1


def gemm_int8_acc(xq: np.ndarray, vals_q: np.ndarray, meta: np.ndarray, k: int) -> np.ndarray:
    """acc = Xq * W'q^T in int64; asserts it fits int32."""
    xq = np.asarray(xq, dtype=np.int64)
    wd = decompress(np.asarray(vals_q, dtype=np.int64), meta, k)
    acc = xq @ wd.T
    if acc.size and (acc.min() < INT32_MIN or acc.max() > INT32_MAX):
        raise OverflowError("int8 GEMM accumulator does not fit int32")
    return acc


def fake_quant(w: np.ndarray, keep: np.ndarray, s_w: np.ndarray) -> np.ndarray:
    """Forward fake-quantisation of the kept weights for Sparse-QAT
    ([Ampere-sparsity] "PTQ and QAT": in the forward pass the weights are
    quantised to int8 and dequantised back to floating point to simulate the
    quantisation; the STE backward and training are not part of this).

    Kept position: bf16_rne(float32(q) * s_w[n]) with q = quantize(w, s_w[n])
    (the same per-channel scale as the int8 inference path); dropped position:
    +0.  Returns bf16 bit patterns [N, K]."""
    w = np.asarray(w, dtype=np.float64)
    keep = np.asarray(keep, dtype=bool)
    s = np.asarray(s_w, dtype=np.float32)[:, None]
    q = quantize(w.astype(np.float32), s).astype(np.float32)
    out = bf16_rne((q * s).astype(np.float32))
    return np.where(keep, out, np.uint16(0)).astype(np.uint16)


def dequant_bf16(acc: np.ndarray, s_x, s_w: np.ndarray) -> np.ndarray:
    """y = bf16_rne(float32(acc) * (s_x * s_w[n])), every step float32 RN.
    Returns bf16 bit patterns [M, N]."""
    c = (np.float32(s_x) * np.asarray(s_w, dtype=np.float32)).astype(np.float32)
    f = np.asarray(acc, dtype=np.int64).astype(np.float32)
    return bf16_rne((f * c[None, :]).astype(np.float32))


def requant_int8(acc: np.ndarray, s_x, s_w: np.ndarray, s_y) -> np.ndarray:
    """int8 output: q = clamp(rint((float32(acc) * (s_x * s_w[n])) / s_y), +-127)."""
    c = (np.float32(s_x) * np.asarray(s_w, dtype=np.float32)).astype(np.float32)
    f = (np.asarray(acc, dtype=np.int64).astype(np.float32) * c[None, :]).astype(np.float32)
    return quantize(f, np.float32(s_y))


# ---------------------------------------------------------------------------
# f2  channel permutation search before masking
#     [Orin ch.7] 3.1 (workflow step 2: search a channel order before the
#     mask is made) and 6.3 (gather the large weights into the same block)
# ---------------------------------------------------------------------------
# Readings (the pages name the goal, not an algorithm):
# * A permutation pi of the K input channels reorders the columns of W (and
#   the same columns of X, so Y is unchanged); the groups of 4 are then
#   pi[0:4], pi[4:8], ...  The objective is the kept score: over every row and
#   every group, the sum of the n_keep largest scores.
# * The search is greedy pairwise swapping: among all pairs of channels that
#   sit in different groups, exchange the pair whose exchange raises the kept
#   score the most; ties go to the pair whose smaller channel index is
#   smallest, then whose larger index is smallest; stop when no exchange
#   raises it or after max_swaps exchanges.
# * So that every comparison is exact, the search runs on integer scores
#   q = rint(s / s_max * 2**24) (float64 divide, round half to even), s as in
#   scores(); an s that is not a finite positive number counts as 0 and
#   s_max = 0 gives q = 0.
PERM_SCALE = 2.0 ** 24
PERM_NO_PAIR = np.iinfo(np.int64).min   # swap_gains entry for a same-group pair


def permutation_scores(w: np.ndarray, mode: str,
                       norms: Optional[np.ndarray] = None) -> np.ndarray:
    """Integer scores q [N, K] (int64) that the permutation search compares."""
    s = scores(w, mode, norms)
    s = np.where(np.isfinite(s) & (s > 0), s, 0.0)
    smax = float(s.max()) if s.size else 0.0
    if smax == 0.0:
        return np.zeros(s.shape, dtype=np.int64)
    return np.rint(s / smax * PERM_SCALE).astype(np.int64)


def _top_sum(groups: np.ndarray, n_keep: int) -> np.ndarray:
    """Sum of the n_keep largest entries along the last axis (size 4)."""
    return np.sort(groups, axis=-1)[..., 4 - n_keep:].sum(axis=-1)


def kept_score(q: np.ndarray, perm: np.ndarray, n_keep: int) -> int:
    """Objective of the permutation search: sum over rows and groups of
    q[:, perm] of the n_keep largest entries of each group of 4."""
    q = np.asarray(q, dtype=np.int64)
    n, k = q.shape
    g = q[:, np.asarray(perm)].reshape(n, k // 4, 4)
    return int(_top_sum(g, n_keep).sum())


def swap_gain(q: np.ndarray, perm: np.ndarray, a: int, b: int, n_keep: int) -> Optional[int]:
    """Change of kept_score when channels a and b trade places, or None when
    they sit in the same group.  Only the two groups involved change."""
    perm = np.asarray(perm)
    pos = np.empty_like(perm)
    pos[perm] = np.arange(perm.size)
    ga, gb = pos[a] // 4, pos[b] // 4
    if ga == gb:
        return None
    old_a = q[:, perm[4 * ga:4 * ga + 4]]
    old_b = q[:, perm[4 * gb:4 * gb + 4]]
    new_a = old_a.copy()
    new_a[:, pos[a] % 4] = q[:, b]
    new_b = old_b.copy()
    new_b[:, pos[b] % 4] = q[:, a]
    return int((_top_sum(new_a, n_keep) + _top_sum(new_b, n_keep)
                - _top_sum(old_a, n_keep) - _top_sum(old_b, n_keep)).sum())


def swap_gains(q: np.ndarray, perm: np.ndarray, n_keep: int) -> np.ndarray:
    """swap_gain for every ordered pair as a [K, K] int64 matrix; pairs in the
    same group (and a == b) hold PERM_NO_PAIR.  Same arithmetic as swap_gain,
    evaluated for all partners b of one channel a at a time."""
    q = np.asarray(q, dtype=np.int64)
    perm = np.asarray(perm)
    n, k = q.shape
    pos = np.empty_like(perm)
    pos[perm] = np.arange(k)
    group = pos // 4
    members = perm.reshape(k // 4, 4)
    kept = _top_sum(q[:, members], n_keep)            # [N, G] kept score per group
    out = np.full((k, k), PERM_NO_PAIR, dtype=np.int64)
    for a in range(k):
        bs = np.flatnonzero(group != group[a])
        if bs.size == 0:
            continue
        new_a = np.repeat(q[:, members[group[a]]][:, None, :], bs.size, axis=1)
        new_a[:, :, pos[a] % 4] = q[:, bs]
        new_b = q[:, members[group[bs]]]              # [N, len(bs), 4]
        new_b[:, np.arange(bs.size), pos[bs] % 4] = q[:, a][:, None]
        gain = (_top_sum(new_a, n_keep).sum(axis=0) + _top_sum(new_b, n_keep).sum(axis=0)
                - kept[:, group[a]].sum() - kept[:, group[bs]].sum(axis=0))
        out[a, bs] = gain
    return out



def permutation_search(q: np.ndarray, n_keep: int, max_swaps: int):
    """Greedy pairwise channel swapping (readings above).

    Returns (perm, swaps, before, after): perm[j] is the channel placed at
    position j, swaps the number of exchanges made, before/after the kept
    score of the identity and of perm."""
    if n_keep not in (2, 3):
        raise ValueError("n_keep must be 2 or 3")
    q = np.asarray(q, dtype=np.int64)
    n, k = q.shape
    if k % 4:
        raise ValueError("K must be a multiple of 4")
    perm = np.arange(k)
    before = kept_score(q, perm, n_keep)
    swaps = 0
    while swaps < max_swaps:
        gains = swap_gains(q, perm, n_keep)
        best = 0
        pair = None
        for a in range(k):                 # first strict maximum in (a, b) order
            for b in range(a + 1, k):
                if gains[a, b] != PERM_NO_PAIR and gains[a, b] > best:
                    best, pair = int(gains[a, b]), (a, b)
        if pair is None:
            break
        a, b = pair
        ia, ib = int(np.flatnonzero(perm == a)[0]), int(np.flatnonzero(perm == b)[0])
        perm[ia], perm[ib] = b, a
        swaps += 1
    return perm, swaps, before, kept_score(q, perm, n_keep)


def _partitions(cols):
    """Every split of the tuple `cols` into unordered groups of 4."""
    if not cols:
        yield []
        return
    first, rest = cols[0], cols[1:]
    for i in range(len(rest)):
        for j in range(i + 1, len(rest)):
            for l in range(j + 1, len(rest)):
                group = (first, rest[i], rest[j], rest[l])
                left = tuple(c for t, c in enumerate(rest) if t not in (i, j, l))
                for tail in _partitions(left):
                    yield [group] + tail


def best_kept_score_bruteforce(q: np.ndarray, n_keep: int) -> int:
    """Largest kept_score over every grouping of the K channels (tiny K
    only: K = 8 has 35 groupings, K = 12 has 5775)."""
    q = np.asarray(q, dtype=np.int64)
    k = q.shape[1]
    best = None
    for groups in _partitions(tuple(range(k))):
        v = kept_score(q, np.array([c for g in groups for c in g]), n_keep)
        best = v if best is None else max(best, v)
    return best


def permute_columns(a: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """A[:, perm]: column j of the result is column perm[j] of A."""
    return np.asarray(a)[:, np.asarray(perm)]


# ---------------------------------------------------------------------------
# f3  3x3 convolution as a GEMM with 2:4 along (kh, kw, Cin)
#     [Orin ch.7] 2.2 A.3 (large 3x3 convolutions, large batch or high
#     resolution, are good candidates) and 2.1 (groups of 4 along the input
#     channels)
# ---------------------------------------------------------------------------
# Readings: stride 1, zero padding 1, NHWC activations X[n][h][w][c], weights
# W[co][kh][kw][c].  The GEMM view has M = n*H*W output pixels, N = Cout and
# K = 9*Cin ordered (kh, kw, c), so a group of 4 runs along Cin inside one tap
# when Cin % 4 == 0; pruning and compression act on W viewed as [Cout][9*Cin].
def conv3x3_nhwc(x: np.ndarray, w4: np.ndarray) -> np.ndarray:
    """y[n,h,w,co] = sum_{kh,kw,c} x[n, h+kh-1, w+kw-1, c] * w4[co,kh,kw,c],
    x zero outside the image; float64.  One matmul per tap."""
    x = np.asarray(x, dtype=np.float64)
    w4 = np.asarray(w4, dtype=np.float64)
    n, hh, ww, c = x.shape
    co = w4.shape[0]
    xp = np.zeros((n, hh + 2, ww + 2, c))
    xp[:, 1:hh + 1, 1:ww + 1, :] = x
    y = np.zeros((n, hh, ww, co))
    for kh in range(3):
        for kw in range(3):
            y += xp[:, kh:kh + hh, kw:kw + ww, :] @ w4[:, kh, kw, :].T
    return y


def conv3x3_weight_as_gemm(w4: np.ndarray) -> np.ndarray:
    """W[co][kh][kw][c] -> [Cout][9*Cin], column (kh*3 + kw)*Cin + c."""
    w4 = np.asarray(w4)
    return w4.reshape(w4.shape[0], -1)


def im2col3x3(x: np.ndarray) -> np.ndarray:
    """A[(n*H + h)*W + w][(kh*3 + kw)*Cin + c] = x[n, h+kh-1, w+kw-1, c]
    (0 outside the image): the GEMM operand of conv3x3_nhwc."""
    x = np.asarray(x)
    n, hh, ww, c = x.shape
    a = np.zeros((n, hh, ww, 9, c), dtype=x.dtype)
    for kh in range(3):
        for kw in range(3):
            dh, dw = kh - 1, kw - 1
            h0, h1 = max(0, -dh), min(hh, hh - dh)
            w0, w1 = max(0, -dw), min(ww, ww - dw)
            a[:, h0:h1, w0:w1, kh * 3 + kw, :] = x[:, h0 + dh:h1 + dh, w0 + dw:w1 + dw, :]
    return a.reshape(n * hh * ww, 9 * c)
