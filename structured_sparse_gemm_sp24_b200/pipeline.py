"""Allocate-and-call helpers over the libsp24 binding.

torch provides the device memory and the current stream; every step runs in
the library's kernels through :mod:`structured_sparse_gemm_sp24_b200.sp24`.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import sp24 as _b

COVERAGE = 0.9999   # "scale covering 99.99 % of the values" (PTQ calibration)


def _u8(nbytes: int, device) -> torch.Tensor:
    # 16 extra bytes keep zero-size requests valid; torch allocations are
    # 256-byte aligned.
    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def colnorm(Xc: torch.Tensor) -> torch.Tensor:
    norms = torch.empty(Xc.shape[1], dtype=torch.float64, device=Xc.device)
    _b.sp24_colnorm(Xc, norms)
    return norms


def prune(W: torch.Tensor, mode: int = _b.SP24_MAGNITUDE, n_keep: int = 2,
          Xc: Optional[torch.Tensor] = None, mask_in: Optional[torch.Tensor] = None,
          workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Keep mask uint8 [N, K/8] (nibble per group, bit p = position p kept)."""
    N, K = W.shape
    mask = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    if mode == _b.SP24_WANDA and workspace is None:
        workspace = _u8(_b.sp24_prune_workspace_bytes(K, mode), W.device)
    _b.sp24_prune(W, Xc, mode, n_keep, mask_in, mask, workspace)
    return mask


def wscale(W: torch.Tensor, mask: torch.Tensor, coverage: float = COVERAGE) -> torch.Tensor:
    s_w = torch.empty(W.shape[0], dtype=torch.float32, device=W.device)
    _b.sp24_wscale(W, mask, coverage, s_w)
    return s_w


def act_scale(X: torch.Tensor, coverage: float = COVERAGE,
              workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    s_x = torch.empty(4, dtype=torch.float32, device=X.device)
    if workspace is None:
        workspace = _u8(_b.sp24_act_scale_workspace_bytes(), X.device)
    _b.sp24_act_scale(X, coverage, s_x, workspace)
    return s_x[:1]


def quantize(X: torch.Tensor, s_x: torch.Tensor) -> torch.Tensor:
    Xq = torch.empty(X.shape, dtype=torch.int8, device=X.device)
    _b.sp24_quantize(X, s_x, Xq)
    return Xq


def alloc_compressed(N: int, K: int, dtype: int, device) -> Tuple[torch.Tensor, torch.Tensor]:
    tdt = torch.bfloat16 if dtype == _b.SP24_BF16 else torch.int8
    vals = torch.empty((N, K // 2), dtype=tdt, device=device)
    meta = _u8(_b.sp24_meta_bytes(N, K), device)
    return vals, meta


def compress(W: torch.Tensor, mask: torch.Tensor, dtype: int = _b.SP24_BF16,
             s_w: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    N, K = W.shape
    vals, meta = alloc_compressed(N, K, dtype, W.device)
    _b.sp24_compress(W, mask, dtype, s_w, vals, meta)
    return vals, meta


def prune_compress(W: torch.Tensor, mode: int = _b.SP24_MAGNITUDE,
                   norms: Optional[torch.Tensor] = None, mask_in: Optional[torch.Tensor] = None,
                   dtype: int = _b.SP24_BF16, s_w: Optional[torch.Tensor] = None,
                   want_mask: bool = False):
    N, K = W.shape
    vals, meta = alloc_compressed(N, K, dtype, W.device)
    mask = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device) if want_mask else None
    _b.sp24_prune_compress(W, mode, norms, mask_in, mask, dtype, s_w, vals, meta)
    return (vals, meta, mask) if want_mask else (vals, meta)


def prune_compress_int8(W: torch.Tensor, coverage: float = COVERAGE, want_mask: bool = False):
    """INT8 weight conversion in one pass: (vals int8, meta, s_w[, mask]) as
    prune (magnitude, 2 of 4) -> wscale -> compress(SP24_INT8) give them."""
    N, K = W.shape
    vals, meta = alloc_compressed(N, K, _b.SP24_INT8, W.device)
    s_w = torch.empty(N, dtype=torch.float32, device=W.device)
    mask = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device) if want_mask else None
    _b.sp24_prune_compress_int8(W, coverage, mask, s_w, vals, meta)
    return (vals, meta, s_w, mask) if want_mask else (vals, meta, s_w)


def prune_progressive(W: torch.Tensor, mode: int = _b.SP24_MAGNITUDE,
                      Xc: Optional[torch.Tensor] = None, compress: bool = True):
    """Progressive pruning in one pass: (mask1 keeping 3 of 4, mask2 keeping 2 of
    4 of the survivors, vals, meta); vals and meta are None without
    compression."""
    N, K = W.shape
    mask1 = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    mask2 = torch.empty((N, K // 8), dtype=torch.uint8, device=W.device)
    vals = meta = None
    if compress:
        vals, meta = alloc_compressed(N, K, _b.SP24_BF16, W.device)
    ws = _u8(max(_b.sp24_prune_workspace_bytes(K, mode), 16), W.device)
    _b.sp24_prune_progressive(W, Xc, mode, mask1, mask2, vals, meta, ws)
    return mask1, mask2, vals, meta


def gemm(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, N: int,
         dtype: int = _b.SP24_BF16, s_x: Optional[torch.Tensor] = None,
         s_w: Optional[torch.Tensor] = None, out_kind: int = _b.SP24_OUT_BF16,
         s_y: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    M = X.shape[0]
    if out is None:
        odt = {_b.SP24_OUT_BF16: torch.bfloat16, _b.SP24_OUT_INT32: torch.int32,
               _b.SP24_OUT_INT8: torch.int8}[out_kind]
        out = torch.empty((M, N), dtype=odt, device=X.device)
    _b.sp24_gemm(X, vals, meta, N, dtype, s_x, s_w, out_kind, s_y, out)
    return out


def fake_quant(W: torch.Tensor, mask: torch.Tensor, s_w: torch.Tensor) -> torch.Tensor:
    """Sparse-QAT forward fake-quantisation of W under `mask` with scales s_w."""
    out = torch.empty_like(W)
    _b.sp24_fake_quant(W, mask, s_w, out)
    return out


def permute_search(W: torch.Tensor, n_keep: int = 2, norms: Optional[torch.Tensor] = None,
                   max_swaps: Optional[int] = None) -> Tuple[torch.Tensor, dict]:
    """Channel order for W before masking (greedy exchange on the kept score).
    Returns (perm int32 [K], {"swaps", "kept_before", "kept_after"})."""
    N, K = W.shape
    ws = _u8(_b.sp24_permute_workspace_bytes(N, K), W.device)
    perm = torch.empty(K, dtype=torch.int32, device=W.device)
    limit = 1 << 40 if max_swaps is None else max_swaps
    res = _b.sp24_permute_search(W, norms, n_keep, limit, perm, ws)
    return perm, res


def permute_columns(A: torch.Tensor, perm: torch.Tensor) -> torch.Tensor:
    """A[:, perm] (the same order applied to W and to the columns of X)."""
    out = torch.empty_like(A)
    _b.sp24_permute_columns(A, perm, out)
    return out


def im2col3x3(X: torch.Tensor) -> torch.Tensor:
    """NHWC X [B, H, W, C] -> the 3x3 convolution's GEMM operand [B*H*W, 9*C]."""
    Bn, H, W, C = X.shape
    A = torch.empty((Bn * H * W, 9 * C), dtype=X.dtype, device=X.device)
    _b.sp24_im2col3x3(X, A)
    return A


def conv3x3(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, Cout: int,
            dtype: int = _b.SP24_BF16, s_x: Optional[torch.Tensor] = None,
            s_w: Optional[torch.Tensor] = None, out_kind: int = _b.SP24_OUT_BF16,
            s_y: Optional[torch.Tensor] = None, path: str = "auto") -> torch.Tensor:
    """3x3 convolution (stride 1, padding 1) of NHWC X with 2:4 weights
    compressed from W[Cout][3][3][C] viewed as [Cout][9*C].  Returns NHWC Y.

    path "implicit": sp24_conv3x3 (token tiles read straight from X);
    "explicit": sp24_im2col3x3 then sp24_gemm; "auto": implicit where its
    tiling rules allow, else explicit."""
    Bn, H, W, _ = X.shape
    odt = {_b.SP24_OUT_BF16: torch.bfloat16, _b.SP24_OUT_INT32: torch.int32,
           _b.SP24_OUT_INT8: torch.int8}[out_kind]
    if path in ("auto", "implicit"):
        y = torch.empty((Bn, H, W, Cout), dtype=odt, device=X.device)
        try:
            _b.sp24_conv3x3(X, vals, meta, Cout, dtype, s_x, s_w, out_kind, s_y, y)
            return y
        except _b.Sp24Error as e:
            if path == "implicit" or e.status not in (_b.SP24_ERR_UNSUPPORTED, _b.SP24_ERR_ALIGN):
                raise
    y = gemm(im2col3x3(X), vals, meta, Cout, dtype, s_x, s_w, out_kind, s_y)
    return y.view(Bn, H, W, Cout)
