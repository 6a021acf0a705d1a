"""Test-side decoder of the metadata operand layout written by sp24_compress.

Independent of the kernels: it restates the tensor-memory metadata layout that
tcgen05.mma.sp reads (2 bits per kept value, one 2048-byte chunk per 128 rows
x 128 K-positions, chunks ordered [row tile][K block]) and maps it back to the
canonical layout (uint8 [N, K/8], nibble = lo | hi << 2, group 2b in the low
nibble of byte b).  A wrong belief here cannot hide a wrong kernel layout: the
GEMM parity tests multiply with the metadata on the tensor cores.

Within a chunk, for chunk row m (0..127) and K-position k (0..127), group
g = k // 4:
* kind::i8 (int8):  the chunk is row-major, 16 bytes per row; group g is
  nibble g % 2 of byte 16*m + g // 2.
* kind::f16 (bf16): each MMA (32 K-positions, j = k // 32) reads one 32-bit
  tensor-memory column; lane L = (m % 8) + 8 * ((k % 32) // 16) + 16 * (m // 16)
  holds rows m and m + 8 of a 16-row block in its low and high half-word,
  4 bits per group in K order.  The chunk stores lane L's 16 bytes at 16*L.
"""
from __future__ import annotations

import numpy as np

BF16, INT8 = 0, 1


def _forward_offsets(dtype: int) -> np.ndarray:
    """offs[m, bb] = byte offset inside a chunk of the canonical byte bb
    (groups 2bb, 2bb+1) of chunk row m."""
    m = np.arange(128)[:, None]
    bb = np.arange(16)[None, :]
    if dtype == INT8:
        return 16 * m + bb
    g = 2 * bb                      # first group of the byte, 0..30 (even)
    k = 4 * g                       # first K-position of that group
    j = k // 32                     # MMA / 32-bit column
    khalf = (k % 32) // 16
    lane = (m % 8) + 8 * khalf + 16 * (m // 16)
    half = (m // 8) % 2             # which half-word of the column
    nib_in_half = (k % 16) // 4     # 0 or 2 for the even group
    return 16 * lane + 4 * j + 2 * half + nib_in_half // 2


def decode(hw: np.ndarray, n: int, k: int, dtype: int) -> np.ndarray:
    """Canonical metadata uint8 [n, k/8] from the chunked operand layout."""
    hw = np.asarray(hw, dtype=np.uint8).ravel()
    kc = (k + 127) // 128
    offs = _forward_offsets(dtype)
    rows = np.arange(n)
    cols = np.arange(k // 8)
    rt, m = rows // 128, rows % 128
    kb, bb = cols // 16, cols % 16
    base = (rt[:, None] * kc + kb[None, :]) * 2048
    return hw[base + offs[m[:, None], bb[None, :]]]


def padding_is_valid(hw: np.ndarray, n: int, k: int, dtype: int) -> bool:
    """Every nibble of the buffer (padding included) is one of the six
    ascending position pairs."""
    hw = np.asarray(hw, dtype=np.uint8).ravel()
    nib = np.concatenate([hw & 0xF, hw >> 4])
    return bool(np.isin(nib, [0x4, 0x8, 0xC, 0x9, 0xD, 0xE]).all())


def is_bijection(dtype: int) -> bool:
    offs = _forward_offsets(dtype).ravel()
    return np.array_equal(np.sort(offs), np.arange(2048))
