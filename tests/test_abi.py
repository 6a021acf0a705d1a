"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/sp24.h declares, answers size queries, and rejects bad
arguments on the host before any CUDA call."""
import ctypes
import os
import re

import numpy as np
import pytest

from structured_sparse_gemm_sp24_b200 import build as sp24_build
from structured_sparse_gemm_sp24_b200 import sp24 as B
from tests import meta_layout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sp24.h")


@pytest.fixture(scope="module")
def lib():
    sp24_build.build()
    return B.lib()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sp24_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n
        assert n in B.SIGNATURES, f"binding lacks {n}"


def test_binding_covers_only_declared_symbols():
    assert set(B.SIGNATURES) == set(_declared_functions())


def test_sizes(lib):
    assert B.sp24_mask_bytes(64, 128) == 64 * 16
    assert B.sp24_mask_bytes(64, 12) == 0
    assert B.sp24_vals_bytes(64, 128, B.SP24_BF16) == 64 * 64 * 2
    assert B.sp24_vals_bytes(64, 128, B.SP24_INT8) == 64 * 64
    # 2 bits per kept value = K/8 bytes per row, rows and K padded to 128
    assert B.sp24_meta_bytes(128, 128) == 2048
    assert B.sp24_meta_bytes(64, 256) == 2 * 2048
    assert B.sp24_meta_bytes(11008, 4096) == 86 * 32 * 2048
    assert B.sp24_meta_bytes(11008, 4096) == 11008 * 4096 // 8
    assert B.sp24_prune_workspace_bytes(768, B.SP24_WANDA) == 768 * 8
    assert B.sp24_prune_workspace_bytes(768, B.SP24_MAGNITUDE) == 0
    assert B.sp24_act_scale_workspace_bytes() >= 2048 * 4
    # storage of the exercise-Q1 row (8 weights, 16-bit): 4 values + 4 bits per group
    assert B.sp24_vals_bytes(1, 8, B.SP24_BF16) * 8 + B.sp24_mask_bytes(1, 8) * 8 == 72


def test_strerror_and_version(lib):
    for code in range(7):
        assert B.strerror(code)
    assert "unknown" in B.strerror(99)
    assert B.sp24_version() >= 100


FAKE = 0x10000   # a 16-byte aligned address that is never dereferenced


def _c(*args):
    return [ctypes.c_void_p(a) if isinstance(a, int) and a >= FAKE else a for a in args]


def test_prune_host_validation(lib):
    f = lib.sp24_prune
    # n_keep outside {2, 3}
    assert f(FAKE, 8, 16, None, 0, B.SP24_MAGNITUDE, 1, None, FAKE, None, None) == B.SP24_ERR_ARG
    # unknown mode
    assert f(FAKE, 8, 16, None, 0, 7, 2, None, FAKE, None, None) == B.SP24_ERR_ARG
    # K not a multiple of 8
    assert f(FAKE, 8, 12, None, 0, B.SP24_MAGNITUDE, 2, None, FAKE, None, None) == B.SP24_ERR_ALIGN
    # misaligned pointer
    assert f(FAKE + 4, 8, 16, None, 0, B.SP24_MAGNITUDE, 2, None, FAKE, None, None) == B.SP24_ERR_ALIGN
    # wanda without calibration rows or workspace
    assert f(FAKE, 8, 16, None, 4, B.SP24_WANDA, 2, None, FAKE, FAKE, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 16, FAKE, 4, B.SP24_WANDA, 2, None, FAKE, None, None) == B.SP24_ERR_ARG
    # null output
    assert f(FAKE, 8, 16, None, 0, B.SP24_MAGNITUDE, 2, None, None, None, None) == B.SP24_ERR_ARG
    # empty problems are a no-op
    assert f(None, 0, 16, None, 0, B.SP24_MAGNITUDE, 2, None, None, None, None) == B.SP24_OK


def test_compress_and_gemm_host_validation(lib):
    c = lib.sp24_compress
    assert c(FAKE, FAKE, 8, 24, B.SP24_BF16, None, FAKE, FAKE, None) == B.SP24_ERR_ALIGN
    assert c(FAKE, FAKE, 8, 48, B.SP24_INT8, FAKE, FAKE, FAKE, None) == B.SP24_ERR_ALIGN
    assert c(FAKE, FAKE, 8, 64, B.SP24_INT8, None, FAKE, FAKE, None) == B.SP24_ERR_ARG
    assert c(FAKE, FAKE, 8, 64, 5, None, FAKE, FAKE, None) == B.SP24_ERR_ARG
    g = lib.sp24_gemm
    # N not a multiple of 8
    assert g(FAKE, 16, 128, FAKE, FAKE, 12, B.SP24_BF16, None, None, B.SP24_OUT_BF16, None,
             FAKE, None) == B.SP24_ERR_ALIGN
    # K too small / not a multiple of 16
    assert g(FAKE, 16, 8, FAKE, FAKE, 16, B.SP24_BF16, None, None, B.SP24_OUT_BF16, None,
             FAKE, None) == B.SP24_ERR_ALIGN
    assert g(FAKE, 16, 40, FAKE, FAKE, 16, B.SP24_BF16, None, None, B.SP24_OUT_BF16, None,
             FAKE, None) == B.SP24_ERR_ALIGN
    # int8 K multiple of 32
    assert g(FAKE, 16, 48, FAKE, FAKE, 16, B.SP24_INT8, FAKE, FAKE, B.SP24_OUT_INT32, None,
             FAKE, None) == B.SP24_ERR_ALIGN
    # bf16 only has a bf16 output; int8 dequant needs the scales
    assert g(FAKE, 16, 128, FAKE, FAKE, 16, B.SP24_BF16, None, None, B.SP24_OUT_INT32, None,
             FAKE, None) == B.SP24_ERR_ARG
    assert g(FAKE, 16, 128, FAKE, FAKE, 16, B.SP24_INT8, None, None, B.SP24_OUT_BF16, None,
             FAKE, None) == B.SP24_ERR_ARG
    assert g(FAKE, 16, 128, FAKE, FAKE, 16, B.SP24_INT8, FAKE, FAKE, B.SP24_OUT_INT8, None,
             FAKE, None) == B.SP24_ERR_ARG
    # int8 output needs N % 16 == 0 (16-byte aligned rows)
    assert g(FAKE, 16, 128, FAKE, FAKE, 24, B.SP24_INT8, FAKE, FAKE, B.SP24_OUT_INT8, FAKE,
             FAKE, None) == B.SP24_ERR_ALIGN
    # empty problems
    assert g(None, 0, 128, None, None, 16, B.SP24_BF16, None, None, B.SP24_OUT_BF16, None,
             None, None) == B.SP24_OK


def test_prune_compress_int8_host_validation(lib):
    f = lib.sp24_prune_compress_int8
    args = lambda n, k, cov, w=FAKE: (w, n, k, ctypes.c_double(cov), None, FAKE, FAKE, FAKE, None)
    assert f(*args(8, 48, 0.9999)) == B.SP24_ERR_ALIGN        # K % 32
    assert f(*args(8, 16, 0.9999)) == B.SP24_ERR_ALIGN        # K < 32
    assert f(*args(8, 64, 0.0)) == B.SP24_ERR_ARG             # coverage outside (0, 1]
    assert f(*args(8, 64, 1.5)) == B.SP24_ERR_ARG
    assert f(*args(-1, 64, 0.9999)) == B.SP24_ERR_ARG
    assert f(*args(8, 64, 0.9999, w=FAKE + 4)) == B.SP24_ERR_ALIGN
    assert f(FAKE, 8, 64, ctypes.c_double(0.9999), None, None, FAKE, FAKE, None) == B.SP24_ERR_ARG
    assert f(*args(0, 64, 0.9999, w=None)) == B.SP24_OK      # empty: a no-op


def test_scale_host_validation(lib):
    assert lib.sp24_wscale(FAKE, FAKE, 8, 16, 0.0, FAKE, None) == B.SP24_ERR_ARG
    assert lib.sp24_wscale(FAKE, FAKE, 8, 16, 1.5, FAKE, None) == B.SP24_ERR_ARG
    assert lib.sp24_act_scale(FAKE, 0, 0.9999, FAKE, FAKE, None) == B.SP24_ERR_ARG
    assert lib.sp24_act_scale(FAKE + 8, 64, 0.9999, FAKE, FAKE, None) == B.SP24_ERR_ALIGN
    assert lib.sp24_quantize(FAKE, -1, FAKE, FAKE, None) == B.SP24_ERR_ARG
    assert lib.sp24_colnorm(FAKE, 4, 12, FAKE, None) == B.SP24_ERR_ALIGN


def test_meta_layout_decoder_is_a_bijection():
    assert meta_layout.is_bijection(meta_layout.BF16)
    assert meta_layout.is_bijection(meta_layout.INT8)


def test_meta_layout_decoder_hand_cases():
    # bf16: chunk row 9 (= row 1 of the second 8-row half), canonical byte 6
    # (groups 12,13 -> K 48..55, MMA 1, second 16-half) -> lane 1 + 8 = 9,
    # column 1, high half-word, first byte: offset 16*9 + 4 + 2 = 150
    hw = np.zeros(2048, dtype=np.uint8)
    hw[150] = 0xAB
    canon = meta_layout.decode(hw, 128, 128, meta_layout.BF16)
    assert canon[9, 6] == 0xAB and canon.sum() == 0xAB
    # int8: row-major
    hw = np.zeros(2048, dtype=np.uint8)
    hw[16 * 9 + 6] = 0xCD
    canon = meta_layout.decode(hw, 128, 128, meta_layout.INT8)
    assert canon[9, 6] == 0xCD and canon.sum() == 0xCD


def test_permute_host_validation(lib):
    ws = lib.sp24_permute_workspace_bytes
    # q and thr (8 N K) + gain (8 K^2) + small pieces
    assert ws(100, 64) >= 8 * 100 * 64 + 8 * 64 * 64
    assert ws(100, 64) < 8 * 100 * 64 + 8 * 64 * 64 + 64 * 100 + 200 * 64 + 4096
    assert ws(0, 64) == 0 and ws(8, 6) == 0 and ws(8, 0) == 0
    assert ws(8, B.SP24_PERMUTE_MAX_K + 4) == 0
    f = lib.sp24_permute_search
    big = 1 << 30
    assert f(FAKE, 8, 16, None, 4, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ARG   # n_keep
    assert f(FAKE, 8, 16, None, 2, -1, FAKE, FAKE, big, None, None) == B.SP24_ERR_ARG   # max_swaps
    assert f(FAKE, 0, 16, None, 2, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ARG   # N
    assert f(None, 8, 16, None, 2, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 16, None, 2, 10, None, FAKE, big, None, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 18, None, 2, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ALIGN  # K % 4
    assert f(FAKE + 2, 8, 16, None, 2, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ALIGN
    assert f(FAKE, 8, 16, FAKE + 8, 2, 10, FAKE, FAKE, big, None, None) == B.SP24_ERR_ALIGN
    assert f(FAKE, 8, 16, None, 2, 10, FAKE, FAKE, ws(8, 16) - 1, None, None) == B.SP24_ERR_ARG
    g = lib.sp24_permute_columns
    assert g(FAKE, 4, 16, 3, FAKE, FAKE + 256, None) == B.SP24_ERR_ARG      # element size
    assert g(FAKE, 4, 16, 2, FAKE, FAKE, None) == B.SP24_ERR_ARG            # in place
    assert g(FAKE, -1, 16, 2, FAKE, FAKE + 256, None) == B.SP24_ERR_ARG
    assert g(FAKE, 0, 16, 2, FAKE, FAKE + 256, None) == B.SP24_OK           # nothing to do
    assert g(FAKE + 4, 4, 16, 2, FAKE, FAKE + 256, None) == B.SP24_ERR_ALIGN
    assert lib.sp24_strerror(B.SP24_ERR_INDEX).decode().startswith("a permutation entry")


def test_im2col_host_validation(lib):
    f = lib.sp24_im2col3x3
    assert f(FAKE, 1, 4, 4, 8, 3, FAKE, None) == B.SP24_ERR_ARG      # element size
    assert f(FAKE, -1, 4, 4, 8, 2, FAKE, None) == B.SP24_ERR_ARG
    assert f(FAKE, 0, 4, 4, 8, 2, FAKE, None) == B.SP24_OK          # nothing to do
    assert f(None, 1, 4, 4, 8, 2, FAKE, None) == B.SP24_ERR_ARG
    assert f(FAKE, 1, 4, 4, 12, 2, FAKE, None) == B.SP24_ERR_ALIGN  # 24-byte pixels
    assert f(FAKE, 1, 4, 4, 8, 1, FAKE, None) == B.SP24_ERR_ALIGN   # 8-byte pixels
    assert f(FAKE + 8, 1, 4, 4, 8, 2, FAKE, None) == B.SP24_ERR_ALIGN


def test_prune_progressive_host_validation(lib):
    f = lib.sp24_prune_progressive
    M, W_ = B.SP24_MAGNITUDE, B.SP24_WANDA
    # no output at all
    assert f(FAKE, 8, 16, None, 0, M, None, None, None, None, None, None) == B.SP24_ERR_ARG
    # values without metadata (or the reverse)
    assert f(FAKE, 8, 16, None, 0, M, FAKE, None, FAKE, None, None, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 16, None, 0, M, FAKE, None, None, FAKE, None, None) == B.SP24_ERR_ARG
    # unknown mode; wanda without calibration rows or workspace
    assert f(FAKE, 8, 16, None, 0, 9, FAKE, None, None, None, None, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 16, None, 4, W_, FAKE, None, None, None, FAKE, None) == B.SP24_ERR_ARG
    assert f(FAKE, 8, 16, FAKE, 4, W_, FAKE, None, None, None, None, None) == B.SP24_ERR_ARG
    # K: multiple of 8 for masks, of 16 with compression
    assert f(FAKE, 8, 12, None, 0, M, FAKE, None, None, None, None, None) == B.SP24_ERR_ALIGN
    assert f(FAKE, 8, 24, None, 0, M, FAKE, FAKE, FAKE, FAKE, None, None) == B.SP24_ERR_ALIGN
    # misaligned pointers
    assert f(FAKE + 2, 8, 16, None, 0, M, FAKE, None, None, None, None, None) == B.SP24_ERR_ALIGN
    assert f(FAKE, 8, 16, None, 0, M, FAKE + 4, None, None, None, None, None) == B.SP24_ERR_ALIGN
    # empty problem
    assert f(None, 0, 16, None, 0, M, None, None, None, None, None, None) == B.SP24_OK


def test_conv3x3_host_validation(lib):
    f = lib.sp24_conv3x3
    BF, I8 = B.SP24_BF16, B.SP24_INT8
    OB, O32, O8 = B.SP24_OUT_BF16, B.SP24_OUT_INT32, B.SP24_OUT_INT8
    ok = (FAKE, 2, 8, 16, 64, FAKE, FAKE, 64, BF, None, None, OB, None, FAKE, None)
    def call(**kw):
        names = ["X", "B", "H", "W", "C", "vals", "meta", "Cout", "dtype", "s_x", "s_w",
                 "out", "s_y", "Y", "stream"]
        a = dict(zip(names, ok))
        a.update(kw)
        return f(*[a[n] for n in names])
    assert call(dtype=5) == B.SP24_ERR_ARG
    assert call(out=O32) == B.SP24_ERR_ARG               # bf16 has only a bf16 output
    assert call(dtype=I8, C=128, out=OB) == B.SP24_ERR_ARG   # dequant needs the scales
    assert call(dtype=I8, C=128, out=O8, s_x=FAKE, s_w=FAKE) == B.SP24_ERR_ARG   # and s_y
    assert call(C=32) == B.SP24_ERR_ALIGN                # 64-byte channel rows
    assert call(dtype=I8, C=64, out=O32) == B.SP24_ERR_ALIGN
    assert call(Cout=60) == B.SP24_ERR_ALIGN
    assert call(X=FAKE + 8) == B.SP24_ERR_ALIGN
    assert call(meta=None) == B.SP24_ERR_ARG
    assert call(B=-1) == B.SP24_ERR_ARG
    assert call(B=0) == B.SP24_OK and call(Cout=0) == B.SP24_OK
