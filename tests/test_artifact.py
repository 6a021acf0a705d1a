"""Compressed-weight files (artifact.py): round trip, header fields and the
errors for files that do not describe their payload.  CPU only: the payload is
arbitrary bytes of the sizes the library computes."""
import struct

import numpy as np
import pytest
import torch

from structured_sparse_gemm_sp24_b200 import artifact as A
from structured_sparse_gemm_sp24_b200 import build as sp24_build
from structured_sparse_gemm_sp24_b200 import sp24 as B


@pytest.fixture(scope="module", autouse=True)
def _lib():
    sp24_build.build()
    B.lib()


def _payload(n, k, dtype, seed=0):
    g = torch.Generator().manual_seed(seed)
    vb, mb = B.sp24_vals_bytes(n, k, dtype), B.sp24_meta_bytes(n, k)
    vals = torch.randint(0, 256, (vb,), dtype=torch.uint8, generator=g)
    vals = vals.view(torch.bfloat16 if dtype == B.SP24_BF16 else torch.int8).view(n, k // 2)
    meta = torch.randint(0, 256, (mb,), dtype=torch.uint8, generator=g)
    s_w = torch.rand(n, generator=g) if dtype == B.SP24_INT8 else None
    return vals, meta, s_w


@pytest.mark.parametrize("n,k,dtype", [(64, 128, B.SP24_BF16), (130, 256, B.SP24_INT8),
                                       (3072, 768, B.SP24_BF16)])
def test_round_trip(tmp_path, n, k, dtype):
    vals, meta, s_w = _payload(n, k, dtype)
    p = str(tmp_path / "w.sp24")
    A.save_compressed(p, vals, meta, n, k, dtype, s_w)
    w = A.load_compressed(p)
    assert (w.n, w.k, w.dtype) == (n, k, dtype)
    assert w.vals.dtype == vals.dtype and w.vals.shape == (n, k // 2)
    assert torch.equal(w.vals.view(torch.uint8), vals.view(torch.uint8))
    assert torch.equal(w.meta, meta)
    if s_w is None:
        assert w.s_w is None
    else:
        assert torch.equal(w.s_w, s_w)


def test_header_fields(tmp_path):
    n, k = 64, 256
    vals, meta, s_w = _payload(n, k, B.SP24_INT8)
    p = tmp_path / "w.sp24"
    A.save_compressed(str(p), vals, meta, n, k, B.SP24_INT8, s_w)
    raw = p.read_bytes()
    magic, fmt, layout, dtype, res, hn, hk, vb, mb, sc = struct.unpack_from("<8sIIIIqqQQQ", raw, 0)
    assert magic == b"SP24W\0\0\0" and fmt == 1 and layout == A.LAYOUT_VERSION and res == 0
    assert (dtype, hn, hk) == (B.SP24_INT8, n, k)
    # int8 values: N*K/2 bytes; metadata: 2 bits per kept value (K/8 bytes a
    # row), rows and K padded to 128; N float32 scales
    assert vb == n * k // 2 and mb == 128 * k // 8 and sc == n
    assert len(raw) == 64 + vb + mb + 4 * sc


def test_rejects_bad_files(tmp_path):
    n, k = 64, 128
    vals, meta, _ = _payload(n, k, B.SP24_BF16)
    p = tmp_path / "w.sp24"
    A.save_compressed(str(p), vals, meta, n, k, B.SP24_BF16)
    raw = bytearray(p.read_bytes())
    bad = tmp_path / "bad.sp24"
    for mutate, what in [(lambda r: r.__setitem__(slice(0, 1), b"X"), "magic"),
                         (lambda r: struct.pack_into("<I", r, 8, 2), "format"),
                         (lambda r: struct.pack_into("<I", r, 12, 7), "layout"),
                         (lambda r: struct.pack_into("<q", r, 24, n + 8), "N"),
                         (lambda r: struct.pack_into("<I", r, 16, 9), "dtype")]:
        r = bytearray(raw)
        mutate(r)
        bad.write_bytes(bytes(r))
        with pytest.raises(ValueError):
            A.load_compressed(str(bad))
    bad.write_bytes(bytes(raw[:-1]))          # truncated payload
    with pytest.raises(ValueError):
        A.load_compressed(str(bad))
    bad.write_bytes(bytes(raw[:40]))          # truncated header
    with pytest.raises(ValueError):
        A.load_compressed(str(bad))


def test_save_checks_sizes(tmp_path):
    n, k = 64, 128
    vals, meta, _ = _payload(n, k, B.SP24_BF16)
    with pytest.raises(ValueError):
        A.save_compressed(str(tmp_path / "a"), vals[:32], meta, n, k, B.SP24_BF16)
    with pytest.raises(ValueError):   # int8 needs scales
        v8, m8, _ = _payload(n, k, B.SP24_INT8)
        A.save_compressed(str(tmp_path / "b"), v8, m8, n, k, B.SP24_INT8, None)
    with pytest.raises(ValueError):   # bf16 takes none
        A.save_compressed(str(tmp_path / "c"), vals, meta, n, k, B.SP24_BF16, torch.ones(n))
