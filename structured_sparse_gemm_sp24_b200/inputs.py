"""Seeded synthetic inputs for the 2:4 sparse workloads.

This module only draws random numbers and casts them to the storage type of
each workload; it holds none of the method's arithmetic (no scoring, no
selection, no packing, no quantisation).  Both the CPU oracle and the CUDA
path are fed from here, so the two sides always see identical bytes.

Recipe (one generator stream per tensor, all from ``torch.Generator`` on the
CPU so that the bytes do not depend on the device):

* weights ``W``: ``randn * sigma`` in fp32, rounded once to bf16 (RNE);
  stream ``seed``.
* activations ``X``: ``randn * sigma`` in fp32, then bf16; stream ``seed+1``.
* calibration activations ``Xc`` (Wanda column norms): stream ``seed+2``.
* long-tail weights (INT8 workload): a Bernoulli(0.01) set of entries drawn
  from stream ``seed+3`` is multiplied by 20 in fp32 before the bf16 cast.
* fp32 activations for the INT8 workload (to be calibrated and quantised by
  the method): ``randn`` in fp32 from stream ``seed+1``, kept in fp32.
* channel-scaled weights (channel permutation search): ``randn * sigma`` times
  a per-input-channel gain ``exp(spread * randn)`` from stream ``seed+4``,
  in fp32 before the single bf16 rounding, so that some channels carry
  larger weights than others, as trained layers do.

The workload names and shapes follow the layer shapes the pages discuss:
a BERT-base FFN fc1 (768 -> 3072), LLM projection shapes (4096 <-> 11008),
square GEMM sweeps and a ResNet bottleneck 1x1 convolution written as a GEMM
over NHWC pixels (2:4 groups along the input channels).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Tuple

import torch


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal_f32(shape: Tuple[int, ...], sigma: float, seed: int) -> torch.Tensor:
    """fp32 samples of N(0, sigma^2) from the CPU generator stream ``seed``."""
    x = torch.randn(shape, generator=_gen(seed), dtype=torch.float32)
    if sigma != 1.0:
        x = x * sigma
    return x


def normal_bf16(shape: Tuple[int, ...], sigma: float, seed: int) -> torch.Tensor:
    """bf16 samples: fp32 N(0, sigma^2) rounded once (RNE) to bf16."""
    return normal_f32(shape, sigma, seed).to(torch.bfloat16)


def long_tail_bf16(shape: Tuple[int, ...], sigma: float, seed: int,
                   tail_seed: int, tail_prob: float = 0.01,
                   tail_gain: float = 20.0) -> torch.Tensor:
    """N(0, sigma^2) weights where a Bernoulli(tail_prob) subset is scaled by
    ``tail_gain`` (in fp32, before the single bf16 rounding)."""
    w = normal_f32(shape, sigma, seed)
    u = torch.rand(shape, generator=_gen(tail_seed), dtype=torch.float32)
    w = torch.where(u < tail_prob, w * tail_gain, w)
    return w.to(torch.bfloat16)


def channel_scaled_bf16(shape: Tuple[int, ...], sigma: float, seed: int,
                        spread: float = 0.5) -> torch.Tensor:
    """[N, K] weights N(0, sigma^2) * exp(spread * g_j), g_j ~ N(0, 1) per input
    channel j from stream ``seed + 4`` (fp32, then one bf16 rounding)."""
    w = normal_f32(shape, sigma, seed)
    g = torch.randn((1, shape[-1]), generator=_gen(seed + 4), dtype=torch.float32)
    return (w * torch.exp(g * spread)).to(torch.bfloat16)


@dataclasses.dataclass
class Workload:
    """One problem instance: tensors are CPU tensors in their storage dtype."""
    name: str
    W: torch.Tensor                     # [N, K] bf16 dense weight
    X: torch.Tensor                     # [M, K] bf16 activations, or fp32 for INT8
    mode: str = "magnitude"             # "magnitude" | "wanda"
    Xc: Optional[torch.Tensor] = None   # [Mc, K] bf16 calibration rows (wanda)
    progressive: bool = False           # prune 3:4 first, then 2:4 on the survivors
    int8: bool = False                  # INT8 path: X is fp32 and is quantised

    @property
    def N(self) -> int:
        return int(self.W.shape[0])

    @property
    def K(self) -> int:
        return int(self.W.shape[1])

    @property
    def M(self) -> int:
        return int(self.X.shape[0])


def tiny(seed: int = 0) -> Workload:
    """W 64x128 ~N(0,1), X 16x128 ~N(0,1), magnitude 2:4."""
    return Workload("tiny_64x128_m16",
                    W=normal_bf16((64, 128), 1.0, seed),
                    X=normal_bf16((16, 128), 1.0, seed + 1))


def bert_fc1(seed: int = 0, M: int = 4096, N: int = 3072, K: int = 768,
             Mc: int = 128) -> Workload:
    """BERT-base FFN fc1: W 3072x768 ~N(0,0.02), Xc 128x768, X 4096x768,
    Wanda score, progressive 3:4 then 2:4."""
    return Workload(f"bert_fc1_wanda_{N}x{K}_m{M}",
                    W=normal_bf16((N, K), 0.02, seed),
                    X=normal_bf16((M, K), 1.0, seed + 1),
                    mode="wanda",
                    Xc=normal_bf16((Mc, K), 1.0, seed + 2),
                    progressive=True)


def llm_proj(N: int, K: int, M: int, seed: int = 0) -> Workload:
    """LLM projection shape, magnitude 2:4, W ~N(0,0.02), X ~N(0,1)."""
    return Workload(f"llm_{N}x{K}_m{M}",
                    W=normal_bf16((N, K), 0.02, seed),
                    X=normal_bf16((M, K), 1.0, seed + 1))


def int8_long_tail(seed: int = 0, M: int = 8192, N: int = 4096,
                   K: int = 4096) -> Workload:
    """INT8 path: W ~N(0,0.02) with 1% of entries x20, fp32 X ~N(0,1)."""
    return Workload(f"int8_{N}x{K}_m{M}",
                    W=long_tail_bf16((N, K), 0.02, seed, seed + 3),
                    X=normal_f32((M, K), 1.0, seed + 1),
                    int8=True)


def square(n: int, seed: int = 0) -> Workload:
    """Square GEMM M=N=K=n, W and X ~N(0,1), magnitude 2:4."""
    return Workload(f"square_{n}",
                    W=normal_bf16((n, n), 1.0, seed),
                    X=normal_bf16((n, n), 1.0, seed + 1))


def conv1x1(batch: int = 64, hw: int = 56, cin: int = 256, cout: int = 64,
            seed: int = 0) -> Workload:
    """ResNet bottleneck 1x1 conv as GEMM over NHWC pixels:
    X [batch*hw*hw, cin], W [cout, cin], 2:4 along cin."""
    M = batch * hw * hw
    return Workload(f"conv1x1_nhwc_{batch}x{hw}x{hw}_{cin}to{cout}",
                    W=normal_bf16((cout, cin), 1.0, seed),
                    X=normal_bf16((M, cin), 1.0, seed + 1))


# The named workloads and their sizes.  The first two are the small case the
# CPU oracle finishes in seconds and the BERT fc1 case; the rest are the LLM,
# INT8 and sweep/conv cases.
LLM_SHAPES = ((11008, 4096), (4096, 11008))
LLM_M = (16, 128, 2048)
SQUARE_SIZES = (1024, 2048, 4096, 8192, 16384)


def all_workload_names() -> Dict[str, str]:
    names = {"tiny": "tiny", "bert_fc1": "bert_fc1", "int8": "int8",
             "conv1x1": "conv1x1"}
    for (n, k) in LLM_SHAPES:
        for m in LLM_M:
            names[f"llm_{n}x{k}_m{m}"] = "llm"
    for s in SQUARE_SIZES:
        names[f"square_{s}"] = "square"
    return names


def by_name(name: str, seed: int = 0) -> Workload:
    """Build a named workload (see ``all_workload_names``)."""
    if name == "tiny":
        return tiny(seed)
    if name == "bert_fc1":
        return bert_fc1(seed)
    if name == "int8":
        return int8_long_tail(seed)
    if name == "conv1x1":
        return conv1x1(seed=seed)
    if name.startswith("llm_"):
        shape, m = name[4:].split("_m")
        n, k = shape.split("x")
        return llm_proj(int(n), int(k), int(m), seed)
    if name.startswith("square_"):
        return square(int(name[7:]), seed)
    raise KeyError(f"unknown workload {name!r}")
