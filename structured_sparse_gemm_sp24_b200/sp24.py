"""Python binding of libsp24 (the C ABI declared in include/sp24.h).

Argument marshalling only: every function takes torch tensors that already
live on the device, checks that they are dense and on CUDA, and passes their
pointers, sizes and the current CUDA stream to the C function of the same
name.  All computation happens in the library's CUDA kernels; there is no
fallback path.  A non-OK status raises :class:`Sp24Error`.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsp24.so")

# enums of include/sp24.h
SP24_OK = 0
SP24_ERR_ARG = 1
SP24_ERR_ALIGN = 2
SP24_ERR_PATTERN = 3
SP24_ERR_CUDA = 4
SP24_ERR_TIMEOUT = 5
SP24_ERR_UNSUPPORTED = 6
SP24_ERR_INDEX = 7
SP24_MAGNITUDE = 0
SP24_WANDA = 1
SP24_BF16 = 0
SP24_INT8 = 1
SP24_OUT_BF16 = 0
SP24_OUT_INT32 = 1
SP24_OUT_INT8 = 2
SP24_NOALLOC_MAX_K = 65536
SP24_PERMUTE_MAX_K = 65536

_c_i64 = ctypes.c_int64
_c_p = ctypes.c_void_p
_c_int = ctypes.c_int
_c_dbl = ctypes.c_double
_c_size = ctypes.c_size_t

# name -> (restype, argtypes)
SIGNATURES = {
    "sp24_mask_bytes": (_c_size, [_c_i64, _c_i64]),
    "sp24_vals_bytes": (_c_size, [_c_i64, _c_i64, _c_int]),
    "sp24_meta_bytes": (_c_size, [_c_i64, _c_i64]),
    "sp24_prune_workspace_bytes": (_c_size, [_c_i64, _c_int]),
    "sp24_colnorm": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p]),
    "sp24_prune": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_int, _c_int, _c_p, _c_p,
                            _c_p, _c_p]),
    "sp24_wscale": (_c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_dbl, _c_p, _c_p]),
    "sp24_act_scale_workspace_bytes": (_c_size, []),
    "sp24_act_scale": (_c_int, [_c_p, _c_i64, _c_dbl, _c_p, _c_p, _c_p]),
    "sp24_quantize": (_c_int, [_c_p, _c_i64, _c_p, _c_p, _c_p]),
    "sp24_compress": (_c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_int, _c_p, _c_p, _c_p, _c_p]),
    "sp24_prune_compress": (_c_int, [_c_p, _c_i64, _c_i64, _c_int, _c_p, _c_p, _c_p, _c_int,
                                     _c_p, _c_p, _c_p, _c_p]),
    "sp24_prune_compress_int8": (_c_int, [_c_p, _c_i64, _c_i64, _c_dbl, _c_p, _c_p, _c_p, _c_p,
                                          _c_p]),
    "sp24_prune_progressive": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_int, _c_p, _c_p,
                                        _c_p, _c_p, _c_p, _c_p]),
    "sp24_conv3x3": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_int,
                              _c_p, _c_p, _c_int, _c_p, _c_p, _c_p]),
    "sp24_gemm": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_p, _c_i64, _c_int, _c_p, _c_p, _c_int,
                           _c_p, _c_p, _c_p]),
    "sp24_device_status": (_c_int, [_c_p]),
    "sp24_strerror": (ctypes.c_char_p, [_c_int]),
    "sp24_version": (_c_int, []),
    "sp24_last_cuda_error": (ctypes.c_char_p, []),
    "sp24_prune_wanda_noalloc": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_i64, _c_int, _c_p, _c_p,
                                          _c_p]),
    "sp24_gemm_plan": (_c_int, [_c_i64, _c_i64, _c_i64, _c_int, _c_p]),
    "sp24_selftest_wait_timeout": (_c_int, [_c_i64, _c_p]),
    "sp24_fake_quant": (_c_int, [_c_p, _c_p, _c_i64, _c_i64, _c_p, _c_p, _c_p]),
    "sp24_permute_workspace_bytes": (_c_size, [_c_i64, _c_i64]),
    "sp24_permute_search": (_c_int, [_c_p, _c_i64, _c_i64, _c_p, _c_int, _c_i64, _c_p, _c_p,
                                     _c_size, _c_p, _c_p]),
    "sp24_permute_columns": (_c_int, [_c_p, _c_i64, _c_i64, _c_int, _c_p, _c_p, _c_p]),
    "sp24_im2col3x3": (_c_int, [_c_p, _c_i64, _c_i64, _c_i64, _c_i64, _c_int, _c_p, _c_p]),
}


class GemmPlan(ctypes.Structure):
    """sp24_gemm_plan_t: the launch sp24_gemm makes for a problem."""
    _fields_ = [("kernel", ctypes.c_char * 16), ("tile_tokens", ctypes.c_int32),
                ("tile_channels", ctypes.c_int32), ("split_k", ctypes.c_int32),
                ("cluster", ctypes.c_int32), ("ctas", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {"kernel": self.kernel.decode(), "tile_tokens": self.tile_tokens,
                "tile_channels": self.tile_channels, "split_k": self.split_k,
                "cluster": self.cluster, "ctas": self.ctas}


class PermuteResult(ctypes.Structure):
    """sp24_permute_result_t."""
    _fields_ = [("swaps", ctypes.c_int64), ("kept_before", ctypes.c_int64),
                ("kept_after", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {"swaps": self.swaps, "kept_before": self.kept_before,
                "kept_after": self.kept_after}


_LIB: Optional[ctypes.CDLL] = None


class Sp24Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        detail = ""
        if self.status == SP24_ERR_CUDA:
            detail = " [" + lib().sp24_last_cuda_error().decode() + "]"
        super().__init__(f"{where}: {strerror(status)} (status {status}){detail}")


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if libsp24.so has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m structured_sparse_gemm_sp24_b200.build` (needs nvcc)")
        h = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(h, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = h
    return _LIB


def strerror(status: int) -> str:
    return lib().sp24_strerror(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != SP24_OK:
        raise Sp24Error(status, where)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("sp24: tensors must be CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("sp24: tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# ------------------------------------------------------------------- sizes
def sp24_mask_bytes(N: int, K: int) -> int:
    return lib().sp24_mask_bytes(N, K)


def sp24_vals_bytes(N: int, K: int, dtype: int) -> int:
    return lib().sp24_vals_bytes(N, K, dtype)


def sp24_meta_bytes(N: int, K: int) -> int:
    return lib().sp24_meta_bytes(N, K)


def sp24_prune_workspace_bytes(K: int, mode: int) -> int:
    return lib().sp24_prune_workspace_bytes(K, mode)


def sp24_act_scale_workspace_bytes() -> int:
    return lib().sp24_act_scale_workspace_bytes()


def sp24_version() -> int:
    return lib().sp24_version()


# ---------------------------------------------------------------- compute
def sp24_colnorm(Xc: torch.Tensor, norms: torch.Tensor, stream=None) -> None:
    Mc, K = Xc.shape
    _check(lib().sp24_colnorm(_ptr(Xc), Mc, K, _ptr(norms), _stream(stream)), "sp24_colnorm")


def sp24_prune(W: torch.Tensor, Xc: Optional[torch.Tensor], mode: int, n_keep: int,
               mask_in: Optional[torch.Tensor], mask_out: torch.Tensor,
               workspace: Optional[torch.Tensor], stream=None) -> None:
    N, K = W.shape
    Mc = 0 if Xc is None else Xc.shape[0]
    _check(lib().sp24_prune(_ptr(W), N, K, _ptr(Xc), Mc, mode, n_keep, _ptr(mask_in),
                            _ptr(mask_out), _ptr(workspace), _stream(stream)), "sp24_prune")


def sp24_prune_wanda_noalloc(W: torch.Tensor, Xc: torch.Tensor, n_keep: int,
                             mask_in: Optional[torch.Tensor], mask_out: torch.Tensor,
                             stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_prune_wanda_noalloc(_ptr(W), N, K, _ptr(Xc), Xc.shape[0], n_keep,
                                          _ptr(mask_in), _ptr(mask_out), _stream(stream)),
           "sp24_prune_wanda_noalloc")


def sp24_wscale(W: torch.Tensor, mask: torch.Tensor, coverage: float, s_w: torch.Tensor,
                stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_wscale(_ptr(W), _ptr(mask), N, K, float(coverage), _ptr(s_w),
                             _stream(stream)), "sp24_wscale")


def sp24_act_scale(X: torch.Tensor, coverage: float, s_x: torch.Tensor,
                   workspace: torch.Tensor, stream=None) -> None:
    _check(lib().sp24_act_scale(_ptr(X), X.numel(), float(coverage), _ptr(s_x),
                                _ptr(workspace), _stream(stream)), "sp24_act_scale")


def sp24_quantize(X: torch.Tensor, s_x: torch.Tensor, Xq: torch.Tensor, stream=None) -> None:
    _check(lib().sp24_quantize(_ptr(X), X.numel(), _ptr(s_x), _ptr(Xq), _stream(stream)),
           "sp24_quantize")


def sp24_compress(W: torch.Tensor, mask: torch.Tensor, dtype: int, s_w: Optional[torch.Tensor],
                  vals: torch.Tensor, meta: torch.Tensor, stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_compress(_ptr(W), _ptr(mask), N, K, dtype, _ptr(s_w), _ptr(vals),
                               _ptr(meta), _stream(stream)), "sp24_compress")


def sp24_prune_compress(W: torch.Tensor, mode: int, norms: Optional[torch.Tensor],
                        mask_in: Optional[torch.Tensor], mask_out: Optional[torch.Tensor],
                        dtype: int, s_w: Optional[torch.Tensor], vals: torch.Tensor,
                        meta: torch.Tensor, stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_prune_compress(_ptr(W), N, K, mode, _ptr(norms), _ptr(mask_in),
                                     _ptr(mask_out), dtype, _ptr(s_w), _ptr(vals), _ptr(meta),
                                     _stream(stream)), "sp24_prune_compress")


def sp24_prune_progressive(W: torch.Tensor, Xc: Optional[torch.Tensor], mode: int,
                           mask1_out: Optional[torch.Tensor], mask2_out: Optional[torch.Tensor],
                           vals: Optional[torch.Tensor], meta: Optional[torch.Tensor],
                           workspace: Optional[torch.Tensor], stream=None) -> None:
    N, K = W.shape
    Mc = Xc.shape[0] if Xc is not None else 0
    _check(lib().sp24_prune_progressive(_ptr(W), N, K, _ptr(Xc), Mc, mode, _ptr(mask1_out),
                                        _ptr(mask2_out), _ptr(vals), _ptr(meta), _ptr(workspace),
                                        _stream(stream)), "sp24_prune_progressive")


def sp24_prune_compress_int8(W: torch.Tensor, coverage: float, mask_out: Optional[torch.Tensor],
                             s_w: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor,
                             stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_prune_compress_int8(_ptr(W), N, K, coverage, _ptr(mask_out), _ptr(s_w),
                                          _ptr(vals), _ptr(meta), _stream(stream)),
           "sp24_prune_compress_int8")


def sp24_conv3x3(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, Cout: int, dtype: int,
                 s_x: Optional[torch.Tensor], s_w: Optional[torch.Tensor], out_kind: int,
                 s_y: Optional[torch.Tensor], Y: torch.Tensor, stream=None) -> None:
    Bn, H, W, C = X.shape
    _check(lib().sp24_conv3x3(_ptr(X), Bn, H, W, C, _ptr(vals), _ptr(meta), Cout, dtype,
                              _ptr(s_x), _ptr(s_w), out_kind, _ptr(s_y), _ptr(Y),
                              _stream(stream)), "sp24_conv3x3")


def sp24_gemm(X: torch.Tensor, vals: torch.Tensor, meta: torch.Tensor, N: int, dtype: int,
              s_x: Optional[torch.Tensor], s_w: Optional[torch.Tensor], out_kind: int,
              s_y: Optional[torch.Tensor], Y: torch.Tensor, stream=None) -> None:
    M, K = X.shape
    _check(lib().sp24_gemm(_ptr(X), M, K, _ptr(vals), _ptr(meta), N, dtype, _ptr(s_x),
                           _ptr(s_w), out_kind, _ptr(s_y), _ptr(Y), _stream(stream)),
           "sp24_gemm")


def sp24_gemm_plan(M: int, N: int, K: int, dtype: int) -> dict:
    """The kernel, tile and grid sp24_gemm uses for an M x N x K problem."""
    plan = GemmPlan()
    _check(lib().sp24_gemm_plan(M, N, K, dtype, ctypes.byref(plan)), "sp24_gemm_plan")
    return plan.as_dict()


def sp24_fake_quant(W: torch.Tensor, mask: torch.Tensor, s_w: torch.Tensor,
                    W_fq: torch.Tensor, stream=None) -> None:
    N, K = W.shape
    _check(lib().sp24_fake_quant(_ptr(W), _ptr(mask), N, K, _ptr(s_w), _ptr(W_fq),
                                 _stream(stream)), "sp24_fake_quant")


def sp24_permute_workspace_bytes(N: int, K: int) -> int:
    return lib().sp24_permute_workspace_bytes(N, K)


def sp24_permute_search(W: torch.Tensor, norms: Optional[torch.Tensor], n_keep: int,
                        max_swaps: int, perm: torch.Tensor, workspace: torch.Tensor,
                        stream=None) -> dict:
    """Greedy channel permutation search; blocks until it has finished."""
    N, K = W.shape
    res = PermuteResult()
    _check(lib().sp24_permute_search(_ptr(W), N, K, _ptr(norms), n_keep, max_swaps, _ptr(perm),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     ctypes.byref(res), _stream(stream)), "sp24_permute_search")
    return res.as_dict()


def sp24_permute_columns(A: torch.Tensor, perm: torch.Tensor, A_out: torch.Tensor,
                         stream=None) -> None:
    rows, K = A.shape
    _check(lib().sp24_permute_columns(_ptr(A), rows, K, A.element_size(), _ptr(perm),
                                      _ptr(A_out), _stream(stream)), "sp24_permute_columns")


def sp24_im2col3x3(X: torch.Tensor, A: torch.Tensor, stream=None) -> None:
    """X NHWC [B][H][W][C] -> A [B*H*W][9*C] (3x3, stride 1, zero padding 1)."""
    Bn, H, W, C = X.shape
    _check(lib().sp24_im2col3x3(_ptr(X), Bn, H, W, C, X.element_size(), _ptr(A),
                                _stream(stream)), "sp24_im2col3x3")


def sp24_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launches the bounded-wait self-test (reports SP24_ERR_TIMEOUT through
    sp24_device_status)."""
    _check(lib().sp24_selftest_wait_timeout(limit_ns, _stream(stream)),
           "sp24_selftest_wait_timeout")


def sp24_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status."""
    return lib().sp24_device_status(_stream(stream))
