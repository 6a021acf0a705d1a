"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each pin is chosen so that a plausible slip in the oracle (a swapped nibble,
a reversed tie-break, a transposed operand, a dropped rounding step) fails at
least one of them:

* the pages' worked examples (tests/golden/worked_examples.json, each cited);
* brute force over every group of the alphabet {-2,-1,-0,0,1,2}^4 with exact
  rational sums, for both n_keep values and both scoring modes;
* algebraic identities: decompress(compress(W)) == W*mask, sparse GEMM ==
  dense GEMM of the masked weight (checked against a pure-Python triple loop
  in exact integers / rationals), progressive 3:4 -> 2:4 == one-shot 2:4;
* library routines for the special cases: torch's float32 -> bfloat16
  rounding, numpy's inverted-CDF quantile.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import sp24_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _bf16(v):
    """Exact float64 value of v rounded to bf16 (RNE) by torch."""
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def _cases():
    with open(GOLDEN) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


# ---------------------------------------------------------------- golden ----
def test_figure_encoding_as_printed():
    c = _cases()["figure_encoding_as_printed"]
    w = _bf16([c["w"]])
    keep = np.array([c["keep"] * 2], dtype=bool)       # K=8: the group twice
    w8 = np.concatenate([w, w], axis=1)
    vals, meta = O.compress(w8, keep)
    assert np.array_equal(vals[0, :2], _bf16(c["vals"]))
    lo, hi = c["codes"]
    assert meta[0, 0] == ((lo | hi << 2) | (lo | hi << 2) << 4)
    # the hardware multiply picks x1 and x3: y = sum of the printed terms
    x = np.array([c["x"] * 2], dtype=np.float64)
    y, _ = O.gemm(x, vals, meta, 8)
    expect = 2 * sum(_bf16([coef])[0] * c["x"][j] for j, coef in c["y_terms"])
    assert y[0, 0] == expect


def test_figure_rule():
    c = _cases()["figure_rule"]
    w = _bf16([c["w"] * 2])
    keep = O.prune(w, O.MAGNITUDE, c["n_keep"])
    assert keep[0, :4].astype(int).tolist() == c["keep"]
    vals, meta = O.compress(w, keep)
    assert meta[0, 0] & 0xF == c["nibble"]
    y, _ = O.gemm(np.array([c["x"] * 2]), vals, meta, 8)
    assert y[0, 0] == 2 * c["y_bf16_weights"]


def test_exercise_q1():
    c = _cases()["exercise_q1"]
    w = _bf16([c["w"]])
    keep = O.prune(w, O.MAGNITUDE, 2)
    assert keep[0].astype(int).tolist() == c["keep"]
    _, meta = O.compress(w, keep)
    assert meta[0, 0] == c["meta_byte"]
    k3 = O.prune(w, O.MAGNITUDE, 3)
    assert k3[0].astype(int).tolist() == c["keep_n3"]
    # storage: 16-bit values, 2 bits per kept value
    dense = 8 * 16
    comp = 4 * 16 + 4 * 2
    assert (dense, comp) == (c["storage_bits_dense"], c["storage_bits_compressed"])
    assert comp / dense == c["storage_ratio"]
    assert O.compress(w.astype(np.float64), keep)[0].size * 16 + meta.size * 8 == comp


def test_exercise_q1_mask_bits():
    w = _bf16([_cases()["exercise_q1"]["w"]])
    keep = O.prune(w, O.MAGNITUDE, 2)
    # mask nibble: bit p = position p kept; group 0 {0,2} -> 0b0101, group 1 {0,1} -> 0b0011
    assert O.pack_mask(keep)[0, 0] == 0b0101 | (0b0011 << 4)
    assert np.array_equal(O.unpack_mask(O.pack_mask(keep), 8), keep)


def test_ties():
    for g in _cases()["ties"]["groups"]:
        w = np.array([g["w"] * 2], dtype=np.float64)
        keep = O.prune(w, O.MAGNITUDE, g["n_keep"])
        assert keep[0, :4].astype(int).tolist() == g["keep"], g
        assert keep[0, 4:].astype(int).tolist() == g["keep"], g


def test_wanda_hand():
    c = _cases()["wanda_hand"]
    xc = np.array(c["xc"], dtype=np.float64)
    assert O.column_norms(xc).tolist() == c["norms"]
    w = _bf16([c["w"]])
    assert O.prune(w, O.WANDA, 2, xc=xc)[0].astype(int).tolist() == c["keep_wanda"]
    assert O.prune(w, O.MAGNITUDE, 2)[0].astype(int).tolist() == c["keep_magnitude"]


def test_int8_round_half_even():
    c = _cases()["int8_round_half_even"]
    w = np.array([c["w"]], dtype=np.float64)
    keep = np.ones_like(w, dtype=bool)
    s = O.channel_scales(w, keep)
    assert s[0] == np.float32(c["scale"])
    assert O.quantize(w, s[:, None])[0].tolist() == c["q"]


# ------------------------------------------------------------ brute force ----
ALPHABET = (-2.0, -1.0, -0.0, 0.0, 1.0, 2.0)


def _brute_keep(s, n_keep):
    """Exact brute force: the kept pair maximises the exact rational score sum,
    ties to the lexicographically smallest pair; for 3 of 4, drop the minimum,
    ties dropping the highest index."""
    fs = [Fraction(v) for v in s]
    if n_keep == 2:
        best = None
        for a, b in itertools.combinations(range(4), 2):
            tot = fs[a] + fs[b]
            if best is None or tot > best[0]:
                best = (tot, (a, b))
        kept = set(best[1])
    else:
        drop = None
        for p in range(4):
            if drop is None or fs[p] <= fs[drop]:
                drop = p
        kept = set(range(4)) - {drop}
    return [int(p in kept) for p in range(4)]


@pytest.mark.parametrize("n_keep", [2, 3])
def test_exhaustive_magnitude(n_keep):
    groups = np.array(list(itertools.product(ALPHABET, repeat=4)), dtype=np.float64)
    w = groups.reshape(1, -1)                      # one row, 1296 groups
    keep = O.prune(w, O.MAGNITUDE, n_keep).reshape(-1, 4)
    for g, kp in zip(groups, keep):
        assert kp.astype(int).tolist() == _brute_keep([abs(v) for v in g], n_keep), g


@pytest.mark.parametrize("n_keep", [2, 3])
def test_exhaustive_wanda(n_keep):
    rng = np.random.default_rng(1)
    groups = np.array(list(itertools.product(ALPHABET, repeat=4)), dtype=np.float64)
    k = groups.size
    # calibration rows with small dyadic entries so the norms are exact
    xc = rng.integers(-3, 4, size=(3, k)).astype(np.float64) / 4
    norms = O.column_norms(xc)
    keep = O.prune(groups.reshape(1, -1), O.WANDA, n_keep, xc=xc).reshape(-1, 4)
    nrm = norms.reshape(-1, 4)
    for g, nr, kp in zip(groups, nrm, keep):
        s = [abs(float(v)) * float(n) for v, n in zip(g, nr)]   # IEEE double products
        assert kp.astype(int).tolist() == _brute_keep(s, n_keep), (g, nr)


def test_exactly_n_keep_per_group_random():
    rng = np.random.default_rng(2)
    w = _bf16(rng.standard_normal((64, 256)).astype(np.float32) * 0.02)
    for n_keep in (2, 3):
        keep = O.prune(w, O.MAGNITUDE, n_keep)
        assert np.all(keep.reshape(64, -1, 4).sum(-1) == n_keep)


def test_group_axis_is_k_not_rows():
    # one row with all its large values in the first group: a row-wise
    # "prune the smaller half" would keep all four, the 2:4 rule keeps two
    w = np.array([[9, 8, 7, 6, 0.1, 0.2, 0.3, 0.4]])
    keep = O.prune(w, O.MAGNITUDE, 2)
    assert keep[0].astype(int).tolist() == [1, 1, 0, 0, 0, 0, 1, 1]


# -------------------------------------------------------------- identities ----
def test_progressive_equals_one_shot():
    rng = np.random.default_rng(3)
    w = _bf16(rng.standard_normal((96, 128)).astype(np.float32) * 0.02)
    xc = _bf16(rng.standard_normal((16, 128)).astype(np.float32))
    for mode, x in ((O.MAGNITUDE, None), (O.WANDA, xc)):
        m1, m2 = O.progressive(w, mode, x)
        assert np.all(m1.reshape(96, -1, 4).sum(-1) == 3)
        assert np.all(m2 <= m1)
        assert np.array_equal(m2, O.prune(w, mode, 2, x))


def test_mask_in_zeroes_scores():
    # a dropped entry scores 0 even when it was the largest
    w = np.array([[5.0, 1.0, 2.0, 3.0, 1, 1, 1, 1]])
    mask_in = np.array([[0, 1, 1, 1, 1, 1, 1, 1]], dtype=bool)
    assert O.prune(w, O.MAGNITUDE, 2, mask_in=mask_in)[0, :4].astype(int).tolist() == [0, 0, 1, 1]


def test_compress_roundtrip_and_pattern_error():
    rng = np.random.default_rng(4)
    w = _bf16(rng.standard_normal((40, 64)).astype(np.float32))
    keep = O.prune(w, O.MAGNITUDE, 2)
    vals, meta = O.compress(w, keep)
    assert vals.shape == (40, 32) and meta.shape == (40, 8)
    assert np.array_equal(O.decompress(vals, meta, 64), np.where(keep, w, 0.0))
    # every nibble is one of the six valid ascending pairs
    nib = np.concatenate([meta & 0xF, meta >> 4], axis=1)
    assert set(np.unique(nib).tolist()) <= {0x4, 0x8, 0xC, 0x9, 0xD, 0xE}
    bad = keep.copy()
    bad[3, 5] = ~bad[3, 5]
    with pytest.raises(O.PatternError):
        O.compress(w, bad)
    with pytest.raises(O.PatternError):
        O.compress(w, O.prune(w, O.MAGNITUDE, 3))


def _py_dense_masked_gemm(x, w, keep):
    """Pure-Python exact triple loop over W*mask (no decompress involved)."""
    m, k = len(x), len(x[0])
    n = len(w)
    y = [[Fraction(0)] * n for _ in range(m)]
    a = [[Fraction(0)] * n for _ in range(m)]
    for i in range(m):
        for j in range(n):
            for t in range(k):
                if keep[j][t]:
                    p = Fraction(x[i][t]) * Fraction(w[j][t])
                    y[i][j] += p
                    a[i][j] += abs(p)
    return y, a


def test_gemm_equals_dense_masked_gemm_exact():
    rng = np.random.default_rng(5)
    m, n, k = 5, 7, 16
    x = rng.integers(-8, 9, size=(m, k)).astype(np.float64) / 8
    w = rng.integers(-16, 17, size=(n, k)).astype(np.float64) / 16
    keep = O.prune(w, O.MAGNITUDE, 2)
    vals, meta = O.compress(w, keep)
    y, a = O.gemm(x, vals, meta, k)
    yr, ar = _py_dense_masked_gemm(x.tolist(), w.tolist(), keep.tolist())
    assert [[Fraction(v) for v in r] for r in y.tolist()] == yr
    assert [[Fraction(v) for v in r] for r in a.tolist()] == ar


def test_gemm_not_transposed():
    # X [M,K] times W'^T: y[m, n] uses row n of W, so swapping operands fails
    x = np.array([[1.0, 0, 0, 0, 0, 0, 0, 0], [0, 0, 0, 0, 1.0, 0, 0, 0]])
    w = np.array([[3.0, 1, 0, 0, 0, 0, 0, 0], [0, 0, 0, 0, 5.0, 1, 0, 0],
                  [7.0, 0, 1, 0, 2.0, 0, 0, 1]])
    keep = O.prune(w, O.MAGNITUDE, 2)
    vals, meta = O.compress(w, keep)
    y, _ = O.gemm(x, vals, meta, 8)
    assert y.tolist() == [[3.0, 0.0, 7.0], [0.0, 5.0, 2.0]]


def test_gemm_float_within_bound():
    rng = np.random.default_rng(6)
    x = _bf16(rng.standard_normal((9, 96)).astype(np.float32))
    w = _bf16(rng.standard_normal((11, 96)).astype(np.float32) * 0.02)
    keep = O.prune(w, O.MAGNITUDE, 2)
    y, a = O.gemm(x, *O.compress(w, keep), 96)
    yr, ar = _py_dense_masked_gemm(x.tolist(), w.tolist(), keep.tolist())
    for i in range(9):
        for j in range(11):
            assert abs(Fraction(y[i, j]) - yr[i][j]) <= Fraction(96) * Fraction(2) ** -52 * ar[i][j]


# ---------------------------------------------------------------- int8 ----
def test_int8_gemm_exact():
    rng = np.random.default_rng(7)
    m, n, k = 4, 6, 32
    xq = rng.integers(-127, 128, size=(m, k)).astype(np.int8)
    wq = rng.integers(-127, 128, size=(n, k)).astype(np.int8)
    keep = O.prune(wq.astype(np.float64), O.MAGNITUDE, 2)
    vals, meta = O.compress(wq, keep)
    assert vals.dtype == np.int8
    acc = O.gemm_int8_acc(xq, vals, meta, k)
    yr, _ = _py_dense_masked_gemm(xq.tolist(), wq.tolist(), keep.tolist())
    assert acc.tolist() == [[int(v) for v in r] for r in yr]


def test_int8_scale_is_row_max_for_small_rows():
    rng = np.random.default_rng(8)
    w = _bf16(rng.standard_normal((16, 4096)).astype(np.float32) * 0.02)
    keep = O.prune(w, O.MAGNITUDE, 2)
    s = O.channel_scales(w, keep)
    rowmax = np.abs(np.where(keep, w, 0)).max(1)
    assert np.array_equal(s, (rowmax.astype(np.float32) / np.float32(127)).astype(np.float32))
    # pruning never drops a group's maximum, so kept-only and all-entries agree
    assert np.array_equal(rowmax, np.abs(w).max(1))


def test_nearest_rank_quantile_vs_numpy():
    rng = np.random.default_rng(9)
    for count in (1, 7, 9999, 10000, 10001, 20011, 123457):
        v = rng.standard_normal(count)
        t = O.quantile_abs(v, 0.9999)
        ref = np.quantile(np.abs(v), 0.9999, method="inverted_cdf")
        assert t == ref, count
    # ranks: c <= 9999 -> the max; ceil(0.9999 * 10000) = 9999 exactly, so
    # c = 10000 and c = 10001 both take the second largest
    assert O.nearest_rank(0.9999, 9999) == 9999
    assert O.nearest_rank(0.9999, 10000) == 9999
    assert O.nearest_rank(0.9999, 10001) == 10000
    v = np.arange(1, 10002, dtype=np.float64)
    assert O.quantile_abs(v, 0.9999) == 10000.0
    assert O.quantile_abs(v[:10000], 0.9999) == 9999.0


def test_tensor_scale_hand_cases():
    # [Ampere-sparsity] "PTQ and QAT": the activation scale covers 99.99 % of
    # the values.  |v| = 1 .. 10001 (signs mixed, order shuffled): the nearest
    # rank is ceil(0.9999 * 10001) = 10000, so t = 10000 and s = 10000 / 127
    # in float32 whatever the signs or the order.
    rng = np.random.default_rng(12)
    mag = np.arange(1, 10002, dtype=np.float64)
    v = rng.permutation(mag * np.where(rng.random(10001) < 0.5, -1.0, 1.0))
    expect = np.float32(np.float32(10000.0) / np.float32(127.0))
    assert O.tensor_scale(v) == expect
    assert O.tensor_scale(v, 0.9999) == expect          # the default coverage is 0.9999
    assert O.tensor_scale(v.reshape(1, -1)) == expect   # layout does not matter
    # all-zero tensor: the quantile is 0 and the scale is 1
    assert O.tensor_scale(np.zeros((3, 5))) == np.float32(1.0)
    assert O.tensor_scale(-np.zeros(7)) == np.float32(1.0)


def test_tensor_scale_ranks_over_every_entry_of_a_matrix():
    # A [3, 6667] matrix of 20001 distinct magnitudes.  The rank over all
    # entries is ceil(0.9999 * 20001) = 19999: the third largest magnitude.
    # Every row (6667 entries, rank 6667) and every column (3 entries, rank 3)
    # takes its own maximum under the same rule, and the fixture places the
    # three largest so that none of those equals the third largest: the
    # largest at (1, 5), the second at (0, 9), the third at (0, 5).
    rows, cols = 3, 6667
    rng = np.random.default_rng(13)
    mags = rng.permutation(np.arange(1, rows * cols - 2, dtype=np.float64))
    x = np.empty((rows, cols))
    slots = [(r, c) for r in range(rows) for c in range(cols)
             if (r, c) not in ((1, 5), (0, 9), (0, 5))]
    for (r, c), m in zip(slots, mags):
        x[r, c] = m
    top = float(rows * cols)
    x[1, 5], x[0, 9], x[0, 5] = top, top - 1, top - 2
    x = x * np.where(rng.random(x.shape) < 0.5, -1.0, 1.0)
    assert O.nearest_rank(0.9999, rows * cols) == rows * cols - 2
    third = np.float32(np.float32(top - 2) / np.float32(127.0))
    assert O.tensor_scale(x) == third
    per_row = {O.tensor_scale(x[r]) for r in range(rows)}
    per_col = {O.tensor_scale(x[:, c]) for c in range(cols)}
    assert third not in per_row and third not in per_col


def test_zero_row_scale_is_one():
    assert O.scale_from_quantile(0.0) == np.float32(1.0)
    w = np.zeros((1, 8))
    keep = O.prune(w, O.MAGNITUDE, 2)
    assert O.channel_scales(w, keep)[0] == 1.0
    assert O.quantize(w, np.float32(1.0)).tolist() == [[0] * 8]


def test_quantize_clamps_and_divides_in_float32():
    v = np.array([1000.0, -1000.0, 126.6, -126.5, 3.0], dtype=np.float32)
    assert O.quantize(v, np.float32(1.0)).tolist() == [127, -127, 127, -126, 3]
    # float32 divide, not float64: choose v, s where the two round differently
    v = np.float32(16777215.0)   # 2^24 - 1
    s = np.float32(3.0)
    assert np.float32(v) / s == np.float32(5592405.0)


def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(10)
    f = rng.standard_normal(200000).astype(np.float32) * np.float32(3.0)
    # exact halfway cases, both parities of the kept lsb
    ties = (rng.integers(0, 1 << 15, 5000, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    near = np.array([np.finfo(np.float32).max, -np.finfo(np.float32).max,
                     1e-40, -1e-40, 0.0, -0.0], dtype=np.float32)
    for arr in (f, ties[np.isfinite(ties)], near):
        mine = O.bf16_rne(arr)
        ref = torch.from_numpy(arr.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(mine, ref)


def test_dequant_order_matches_torch_float32():
    rng = np.random.default_rng(11)
    acc = rng.integers(-(1 << 24), 1 << 24, size=(8, 16))
    acc[0, 0] = (1 << 24) + 1            # int -> float32 rounds here
    s_x = np.float32(0.0123)
    s_w = rng.uniform(1e-4, 1e-2, 16).astype(np.float32)
    mine = O.dequant_bf16(acc, s_x, s_w)
    c = torch.tensor(s_x) * torch.from_numpy(s_w)
    ref = (torch.from_numpy(acc).to(torch.float32) * c[None, :]).to(torch.bfloat16)
    assert np.array_equal(mine, ref.view(torch.int16).numpy().view(np.uint16))
    # hand value: 3 * (0.5 * 0.25) = 0.375 = 0x3EC0 in bf16
    assert O.dequant_bf16(np.array([[3]]), np.float32(0.5), np.array([0.25], np.float32))[0, 0] == 0x3EC0
    assert O.bf16_bits_to_f64(np.array([0x3EC0]))[0] == 0.375


def test_requant_int8():
    acc = np.array([[100, -100, 3, 1000000]])
    q = O.requant_int8(acc, np.float32(0.5), np.array([0.5, 0.5, 0.5, 0.5], np.float32), np.float32(2.0))
    # 100*0.25/2 = 12.5 -> 12 (half even); -12.5 -> -12; 0.375 -> 0; clamp
    assert q.tolist() == [[12, -12, 0, 127]]


def test_column_norms_exact_and_sequential():
    # Pythagorean columns: exact norms
    xc = np.array([[3.0, 5.0, 8.0], [4.0, 12.0, 15.0]])
    assert O.column_norms(xc).tolist() == [5.0, 13.0, 17.0]
    # the float64 sum runs in token order: 32 squares of 2^-27 (2^-54 each)
    # survive when they come before the 1, and are each lost after it
    small_first = np.array([[2.0 ** -27]] * 32 + [[1.0]])
    big_first = np.array([[1.0]] + [[2.0 ** -27]] * 32)
    assert O.column_norms(small_first)[0] == 1.0 + 2.0 ** -50
    assert O.column_norms(big_first)[0] == 1.0
    assert math.sqrt(1.0 + 2.0 ** -49) == 1.0 + 2.0 ** -50


def test_wanda_prune_uses_input_columns():
    # the score multiplies W[n, j] by the norm of input feature j (column j of
    # Xc), not by a per-row or per-output statistic
    w = np.array([[1.0, 1.0, 1.0, 1.0], [1.0, 1.0, 1.0, 1.0]] * 1)
    w = np.concatenate([w, w], axis=1)
    xc = np.zeros((1, 8))
    xc[0, 2] = 4.0
    xc[0, 3] = 2.0
    xc[0, 4] = 1.0
    keep = O.prune(w, O.WANDA, 2, xc=xc)
    assert keep[:, :4].astype(int).tolist() == [[0, 0, 1, 1]] * 2
    assert keep[:, 4:].astype(int).tolist() == [[1, 1, 0, 0]] * 2


# --------------------------------------------------------- Sparse-QAT fake quant
def _bits_to_f32(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32)


def test_fake_quant_round_trips_exact_multiples():
    # w = k * s with s a power of two and |k| <= 127: quantise -> dequantise
    # must give w back exactly (k * s is exact in bf16 for |k| < 256)
    s = np.float32(2.0 ** -5)
    k = np.arange(-127, 128, dtype=np.float64)
    w = (k * float(s))[None, :].repeat(2, 0)
    w = np.concatenate([w, np.zeros((2, 1))], axis=1)          # K = 256
    keep = np.ones_like(w, dtype=bool)
    got = _bits_to_f32(O.fake_quant(w, keep, np.array([s, s], dtype=np.float32)))
    assert np.array_equal(got.astype(np.float64), w)


def test_fake_quant_clamps_ties_and_drops():
    s = np.float32(0.25)
    w = np.array([[200 * 0.25, -200 * 0.25, 2.5 * 0.25, 3.5 * 0.25, -2.5 * 0.25, 0.5 * 0.25,
                   1.0, 1.0]])
    keep = np.array([[1, 1, 1, 1, 1, 1, 0, 1]], dtype=bool)
    got = _bits_to_f32(O.fake_quant(w, keep, np.array([s], dtype=np.float32)))[0]
    # clamp to +-127 s; half-integer quotients round to even: 2.5 -> 2, 3.5 -> 4,
    # -2.5 -> -2, 0.5 -> 0; a dropped position is +0
    assert list(got) == [127 * 0.25, -127 * 0.25, 0.5, 1.0, -0.5, 0.0, 0.0, 1.0]
    assert O.fake_quant(w, keep, np.array([s], dtype=np.float32))[0, 6] == 0   # +0 bits


# ------------------------------------------------- channel permutation search
# [Orin ch.7] 3.1 step 2 and 6.3: search a channel order before masking so
# that large weights share groups.  The greedy rule and the integer scores are
# readings (see the oracle); the hand-derived cases below follow them step by
# step, and brute force over every grouping bounds the result.

def test_perm_scores_scale_round_half_even_and_edges():
    big = float(2 ** 24)
    q = O.permutation_scores(np.array([[big, -big / 2, 0.5, 1.5, 2.5, -0.0, 3.0, 0.0]]),
                             O.MAGNITUDE)
    # s / s_max * 2^24 = s here; 0.5 -> 0, 1.5 -> 2, 2.5 -> 2 (half to even)
    assert q.tolist() == [[2 ** 24, 2 ** 23, 0, 2, 2, 0, 3, 0]]
    assert not O.permutation_scores(np.zeros((3, 8)), O.MAGNITUDE).any()
    q = O.permutation_scores(np.array([[np.nan, np.inf, 4.0, -2.0]]), O.MAGNITUDE)
    assert q.tolist() == [[0, 0, 2 ** 24, 2 ** 23]]
    q = O.permutation_scores(np.array([[1.0, -1.0, 2.0, 1.0]]), O.WANDA,
                             norms=np.array([4.0, 2.0, 1.0, 0.0]))
    assert q.tolist() == [[2 ** 24, 2 ** 23, 2 ** 23, 0]]


def test_perm_hand_example_two_of_four():
    # One row [9 9 9 9 | 0 0 0 0].  Step 1: every (a in 0..3, b in 4..7)
    # moves a 9 into the empty group, gain 9; the lowest pair (0, 4) wins.
    # Step 2: groups {0,9,9,9 | 9,0,0,0}; moving one more 9 across gains 9
    # ((1, 5) is the lowest such pair); swapping 9 for 9 gains 0 and moving
    # the 9 back loses 9.  Step 3: every swap gains <= 0, stop.
    q = O.permutation_scores(np.array([[9, 9, 9, 9, 0, 0, 0, 0]], float), O.MAGNITUDE)
    perm, swaps, before, after = O.permutation_search(q, 2, 100)
    assert perm.tolist() == [4, 5, 2, 3, 0, 1, 6, 7]
    assert (swaps, before, after) == (2, 2 * 2 ** 24, 4 * 2 ** 24)
    perm1, swaps1, _, after1 = O.permutation_search(q, 2, 1)
    assert perm1.tolist() == [4, 1, 2, 3, 0, 5, 6, 7] and (swaps1, after1) == (1, 3 * 2 ** 24)
    assert O.best_kept_score_bruteforce(q, 2) == after


def test_perm_hand_example_three_of_four():
    # One row [4 3 2 1 | 8 7 6 5], keep 3: kept 9 + 21 = 30.  The best
    # grouping drops the two smallest values (1 and 2) from different groups:
    # 36 - 3 = 33, so no swap gains more than 3.  Pairs (0, *) gain 1 and
    # (1, *) gain 2; (2, 4) gives {4,3,8,1 | 2,7,6,5} = 15 + 18 = 33, the
    # first pair with gain 3.  Units: q = v * 2^24 / 8 = v * 2^21.
    q = O.permutation_scores(np.array([[4, 3, 2, 1, 8, 7, 6, 5]], float), O.MAGNITUDE)
    perm, swaps, before, after = O.permutation_search(q, 3, 100)
    assert perm.tolist() == [0, 1, 4, 3, 2, 5, 6, 7]
    assert (swaps, before, after) == (1, 30 * 2 ** 21, 33 * 2 ** 21)
    assert O.best_kept_score_bruteforce(q, 3) == 33 * 2 ** 21
    g = O.swap_gains(q, np.arange(8), 3)
    assert [g[0, b] for b in range(4, 8)] == [2 ** 21] * 4
    assert [g[1, b] for b in range(4, 8)] == [2 * 2 ** 21] * 4
    assert g[2, 4] == 3 * 2 ** 21


def test_perm_pages_row_is_already_optimal():
    # The 1x4 row [0.9 0.1 0.9 0.1] that [Orin ch.7] 3.1 uses to motivate the
    # permutation already keeps both 0.9 under the keep-the-largest rule; no
    # exchange can raise the kept score, so the search leaves the order alone.
    q = O.permutation_scores(np.array([[0.9, 0.1, 0.9, 0.1] * 2]), O.MAGNITUDE)
    perm, swaps, before, after = O.permutation_search(q, 2, 100)
    assert perm.tolist() == list(range(8)) and swaps == 0 and before == after
    assert O.best_kept_score_bruteforce(q, 2) == before


@pytest.mark.parametrize("n_keep", [2, 3])
def test_perm_gains_equal_full_rescore(n_keep):
    rng = np.random.default_rng(11 + n_keep)
    q = rng.integers(0, 6, size=(5, 12)).astype(np.int64)   # small range: many ties
    for perm in (np.arange(12), rng.permutation(12)):
        g = O.swap_gains(q, perm, n_keep)
        base = O.kept_score(q, perm, n_keep)
        pos = np.argsort(perm)
        for a in range(12):
            for b in range(12):
                if pos[a] // 4 == pos[b] // 4:
                    assert g[a, b] == O.PERM_NO_PAIR and O.swap_gain(q, perm, a, b, n_keep) is None
                    continue
                p2 = perm.copy()
                p2[pos[a]], p2[pos[b]] = b, a
                want = O.kept_score(q, p2, n_keep) - base
                assert g[a, b] == want == O.swap_gain(q, perm, a, b, n_keep)


def test_perm_partition_enumeration_is_complete():
    for k, count in ((4, 1), (8, 35), (12, 5775)):
        seen = set()
        for groups in O._partitions(tuple(range(k))):
            assert sorted(c for g in groups for c in g) == list(range(k))
            seen.add(frozenset(frozenset(g) for g in groups))
        # K! / ((4!)^(K/4) * (K/4)!) groupings, each produced once
        assert len(seen) == count == math.factorial(k) // (
            math.factorial(4) ** (k // 4) * math.factorial(k // 4))


@pytest.mark.parametrize("n_keep", [2, 3])
@pytest.mark.parametrize("k", [8, 12])
def test_perm_search_is_a_local_optimum_under_the_bruteforce_bound(n_keep, k):
    rng = np.random.default_rng(100 * k + n_keep)
    for trial in range(3):
        w = rng.standard_normal((4, k)) * rng.uniform(0.2, 3.0, size=k)
        q = O.permutation_scores(w, O.MAGNITUDE)
        perm, swaps, before, after = O.permutation_search(q, n_keep, 1000)
        assert sorted(perm.tolist()) == list(range(k))
        assert before == O.kept_score(q, np.arange(k), n_keep)
        assert after == O.kept_score(q, perm, n_keep)
        assert before + swaps <= after <= O.best_kept_score_bruteforce(q, n_keep)
        pos = np.argsort(perm)
        for a in range(k):                        # no single exchange improves
            for b in range(a + 1, k):
                if pos[a] // 4 != pos[b] // 4:
                    p2 = perm.copy()
                    p2[pos[a]], p2[pos[b]] = b, a
                    assert O.kept_score(q, p2, n_keep) <= after


def test_perm_columns_leave_the_product_unchanged():
    # The exchange is an equivalent transform: permuting the same input
    # channels of X and W leaves Y = X W^T unchanged (exact in integers).
    rng = np.random.default_rng(5)
    x = rng.integers(-9, 10, size=(6, 16))
    w = rng.integers(-9, 10, size=(5, 16))
    perm = rng.permutation(16)
    xp, wp = O.permute_columns(x, perm), O.permute_columns(w, perm)
    assert (xp @ wp.T == x @ w.T).all()
    assert (xp[:, np.argsort(perm)] == x).all()


# ------------------------------------------------- 3x3 convolution as a GEMM
# [Orin ch.7] 2.2 A.3 and 2.1: stride 1, zero padding 1, NHWC, groups of 4
# along (kh, kw, Cin).

def _conv3x3_loops(x, w4):
    """Seven nested loops over integers, bounds checked per term."""
    n, hh, ww, c = x.shape
    co = w4.shape[0]
    y = [[[[0] * co for _ in range(ww)] for _ in range(hh)] for _ in range(n)]
    for b in range(n):
        for h in range(hh):
            for w in range(ww):
                for o in range(co):
                    s = 0
                    for kh in range(3):
                        for kw in range(3):
                            ih, iw = h + kh - 1, w + kw - 1
                            if 0 <= ih < hh and 0 <= iw < ww:
                                for ci in range(c):
                                    s += int(x[b, ih, iw, ci]) * int(w4[o, kh, kw, ci])
                    y[b][h][w][o] = s
    return np.array(y, dtype=np.float64)


def test_conv3x3_equals_bruteforce_and_im2col_gemm():
    rng = np.random.default_rng(31)
    x = rng.integers(-4, 5, size=(2, 4, 5, 8))
    w4 = rng.integers(-4, 5, size=(3, 3, 3, 8))
    want = _conv3x3_loops(x, w4)
    assert np.array_equal(O.conv3x3_nhwc(x, w4), want)
    a = O.im2col3x3(x)
    assert a.shape == (2 * 4 * 5, 72)
    assert np.array_equal((a @ O.conv3x3_weight_as_gemm(w4).T).reshape(want.shape), want)


def test_conv3x3_special_kernels():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((1, 4, 3, 4))
    # centre tap only: a 1x1 convolution
    w4 = np.zeros((5, 3, 3, 4))
    w4[:, 1, 1, :] = rng.standard_normal((5, 4))
    assert np.allclose(O.conv3x3_nhwc(x, w4), x @ w4[:, 1, 1, :].T, rtol=0, atol=1e-15)
    # top-left tap with the identity over channels: y[h][w] = x[h-1][w-1]
    w4 = np.zeros((4, 3, 3, 4))
    w4[:, 0, 0, :] = np.eye(4)
    y = O.conv3x3_nhwc(x, w4)
    assert (y[:, 0, :, :] == 0).all() and (y[:, :, 0, :] == 0).all()
    assert np.array_equal(y[:, 1:, 1:, :], x[:, :-1, :-1, :])


def test_im2col_columns_follow_taps_then_channels():
    x = np.arange(1, 1 + 2 * 2 * 8).reshape(1, 2, 2, 8)
    a = O.im2col3x3(x)
    # pixel (0, 0): taps with kh = 0 or kw = 0 read outside the image
    assert (a[0, :8 * 4] == 0).all()              # taps (0,0) (0,1) (0,2) (1,0)
    assert (a[0, 4 * 8:5 * 8] == x[0, 0, 0]).all()  # tap (1,1) = the pixel itself
    assert (a[0, 5 * 8:6 * 8] == x[0, 0, 1]).all()  # tap (1,2) = right neighbour
    assert (a[0, 8 * 8:9 * 8] == x[0, 1, 1]).all()  # tap (2,2) = down-right
    # pixel (1, 1) (row 3): tap (0,0) = x[0,0]
    assert (a[3, 0:8] == x[0, 0, 0]).all()


def test_sparse_conv3x3_groups_stay_inside_one_tap():
    rng = np.random.default_rng(33)
    x = rng.integers(-3, 4, size=(1, 3, 4, 8))
    w4 = rng.integers(-3, 4, size=(4, 3, 3, 8)).astype(np.float64)
    wg = O.conv3x3_weight_as_gemm(w4)
    keep = O.prune(wg, O.MAGNITUDE, 2)
    # with Cin % 4 == 0 every group of 4 columns lies in one (kh, kw) tap
    for g in range(wg.shape[1] // 4):
        assert len({(4 * g + i) // 8 for i in range(4)}) == 1
    w4m = np.where(keep, wg, 0.0).reshape(w4.shape)
    want = _conv3x3_loops(x, w4m.astype(np.int64))
    vals, meta = O.compress(wg, keep)
    got, _ = O.gemm(O.im2col3x3(x).astype(np.float64), vals, meta, wg.shape[1])
    assert np.array_equal(got.reshape(want.shape), want)
