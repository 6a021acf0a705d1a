"""Files holding a compressed 2:4 weight, so that pruning and compression run
once offline and inference only loads the result ([Sparse-accel forum]
(oeforum.com): the sparse weight is converted offline, once; [Ampere-sparsity]
Figure 1: the values plus their index metadata are what inference needs).

Layout (little-endian): a 64-byte header, then the values, the metadata and,
for int8, the per-output-channel scales.

    offset  size  field
    0       8     magic b"SP24W\\0\\0\\0"
    8       4     format version (1)
    12      4     metadata layout version (LAYOUT_VERSION: the tcgen05.mma.sp
                  operand layout this library's kernels write and read)
    16      4     dtype (sp24.SP24_BF16 or sp24.SP24_INT8)
    20      4     reserved (0)
    24      8     N (output channels, rows of W)
    32      8     K (input channels)
    40      8     values bytes   (sp24_vals_bytes(N, K, dtype))
    48      8     metadata bytes (sp24_meta_bytes(N, K))
    56      8     scale count    (N for int8, 0 for bf16)

Loading checks every field against what the library computes for N, K and
dtype and raises ValueError on any mismatch (a file written for another
layout, a truncated file, a header that does not describe its payload).
"""
from __future__ import annotations

import os
import struct
from typing import NamedTuple, Optional

import torch

from . import sp24 as _b

MAGIC = b"SP24W\0\0\0"
FORMAT_VERSION = 1
LAYOUT_VERSION = 1
_HEADER = struct.Struct("<8sIIIIqqQQQ")
assert _HEADER.size == 64


class CompressedWeight(NamedTuple):
    vals: torch.Tensor              # bf16 or int8 [N, K/2]
    meta: torch.Tensor              # uint8 [sp24_meta_bytes(N, K)]
    s_w: Optional[torch.Tensor]     # float32 [N] for int8, else None
    n: int
    k: int
    dtype: int


def _expect(n: int, k: int, dtype: int):
    if dtype not in (_b.SP24_BF16, _b.SP24_INT8):
        raise ValueError(f"unknown dtype {dtype}")
    if n < 1 or k < 16 or k % (16 if dtype == _b.SP24_BF16 else 32) != 0:
        raise ValueError(f"bad shape N={n}, K={k} for dtype {dtype}")
    vb = _b.sp24_vals_bytes(n, k, dtype)
    mb = _b.sp24_meta_bytes(n, k)
    sc = n if dtype == _b.SP24_INT8 else 0
    return vb, mb, sc


def save_compressed(path: str, vals: torch.Tensor, meta: torch.Tensor, n: int, k: int,
                    dtype: int, s_w: Optional[torch.Tensor] = None) -> None:
    """Writes the compressed weight (any device) to `path`."""
    vb, mb, sc = _expect(n, k, dtype)
    got_v = vals.numel() * vals.element_size()
    got_m = meta.numel() * meta.element_size()
    if got_v != vb or got_m != mb:
        raise ValueError(f"sizes {got_v}/{got_m} bytes, expected {vb}/{mb} for N={n}, K={k}")
    if (s_w is None) != (sc == 0) or (s_w is not None and s_w.numel() != sc):
        raise ValueError("int8 weights need their N float32 scales, bf16 weights none")
    hdr = _HEADER.pack(MAGIC, FORMAT_VERSION, LAYOUT_VERSION, dtype, 0, n, k, vb, mb, sc)
    tmp = path + ".tmp"
    with open(tmp, "wb") as f:
        f.write(hdr)
        f.write(vals.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes())
        f.write(meta.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes())
        if s_w is not None:
            f.write(s_w.detach().to(torch.float32).contiguous().cpu().numpy().tobytes())
    os.replace(tmp, path)


def load_compressed(path: str, device="cpu") -> CompressedWeight:
    """Reads a file written by save_compressed; tensors land on `device`."""
    with open(path, "rb") as f:
        raw = f.read()
    if len(raw) < _HEADER.size:
        raise ValueError("file shorter than the header")
    magic, fmt, layout, dtype, _res, n, k, vb, mb, sc = _HEADER.unpack_from(raw, 0)
    if magic != MAGIC:
        raise ValueError("not a compressed 2:4 weight file")
    if fmt != FORMAT_VERSION:
        raise ValueError(f"format version {fmt}, this library reads {FORMAT_VERSION}")
    if layout != LAYOUT_VERSION:
        raise ValueError(f"metadata layout {layout}, this library uses {LAYOUT_VERSION}")
    evb, emb, esc = _expect(n, k, dtype)
    if (vb, mb, sc) != (evb, emb, esc):
        raise ValueError(f"header sizes {vb}/{mb}/{sc} do not match N={n}, K={k}")
    total = _HEADER.size + vb + mb + 4 * sc
    if len(raw) != total:
        raise ValueError(f"file is {len(raw)} bytes, header describes {total}")
    buf = torch.frombuffer(bytearray(raw), dtype=torch.uint8)
    o = _HEADER.size
    vals = buf[o:o + vb].clone()
    o += vb
    meta = buf[o:o + mb].clone()
    o += mb
    vals = vals.view(torch.bfloat16 if dtype == _b.SP24_BF16 else torch.int8).view(n, k // 2)
    s_w = buf[o:o + 4 * sc].clone().view(torch.float32) if sc else None
    dev = torch.device(device)
    return CompressedWeight(vals.to(dev), meta.to(dev), None if s_w is None else s_w.to(dev),
                            n, k, dtype)
