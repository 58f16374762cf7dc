"""Seeded synthetic inputs for the block-scaled W8A8 linear layer and MoE.

This module is shared by the CUDA path's tests/benchmark and by the CPU
oracle's tests.  It holds NO arithmetic of the quantisation method: it only
draws Gaussian activations and weights, picks outlier channels, and builds MoE
routing (softmax + top-k, a harness choice; the library receives the expert
ids and weights as inputs).

Workloads (the shapes and distributions of the pages' block-wise INT8 and
blockwise FP8 linear layers, restated as synthetic inputs):

  tiny     A bf16 [16, 200] ~ N(0,1), 2 outlier channels x20;
           W fp32 [320, 200] ~ N(0, 0.02); blocks [128, 128]; seed 0
  decode   M in {1, 8, 32, 64}; N = K = 4096; A ~ N(0,1) + 1% outlier channels
           (41 of 4096) x30; W ~ N(0, 0.02); seeds 1..4
  prefill  M = 4096, N = 14336, K = 4096; W ~ N(0, 0.015); A as decode; seed 5
  fp8      M = 2048, N = 4096, K = 14336; W ~ N(0, 0.01) (e4m3);
           A ~ N(0,1); seed 6
  moe      T = 4096, H = 4096, E = 8, top-2 from softmax of N(0,1) logits;
           w13 [8, 28672, 4096], w2 [8, 4096, 14336] ~ N(0, 0.015); seed 7
  perchannel  the prefill shape with block_n = 1, block_k = K (per-token and
           per-channel scales); seed 8
  mxfp8    the FP8 shape, MXFP8 (1 x 32 groups, E8M0 scales) on both operands;
           W ~ N(0, 0.01); seed 9

Generators use torch.Generator so that the same recipe runs on the CPU (for
oracle comparisons) or directly on a CUDA device (for large benchmarks).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

INT8 = 0
FP8 = 1
MXFP8 = 2        # workload marker: 32-element E8M0-scaled e4m3 groups


@dataclasses.dataclass(frozen=True)
class Linear:
    name: str
    M: int
    N: int
    K: int
    w_std: float
    n_outliers: int
    outlier_scale: float
    dtype: int
    seed: int
    block_n: int = 128
    block_k: int = 128


@dataclasses.dataclass(frozen=True)
class MoE:
    name: str
    T: int
    H: int
    I: int
    E: int
    topk: int
    w_std: float
    seed: int
    dtype: int = INT8
    block_n: int = 128
    block_k: int = 128


def one_percent(K: int) -> int:
    return int(round(0.01 * K))


TINY = Linear("tiny_int8_m16_n320_k200", 16, 320, 200, 0.02, 2, 20.0, INT8, 0)
DECODE_MS = (1, 8, 32, 64)
DECODE = tuple(
    Linear(f"decode_int8_m{m}_n4096_k4096", m, 4096, 4096, 0.02, one_percent(4096), 30.0,
           INT8, 1 + i) for i, m in enumerate(DECODE_MS))
PREFILL = Linear("prefill_int8_m4096_n14336_k4096", 4096, 14336, 4096, 0.015,
                 one_percent(4096), 30.0, INT8, 5)
FP8_LINEAR = Linear("fp8_e4m3_m2048_n4096_k14336", 2048, 4096, 14336, 0.01, 0, 1.0, FP8, 6)
MOE = MoE("moe_int8_t4096_h4096_i14336_e8_top2", 4096, 4096, 14336, 8, 2, 0.015, 7)
# the degenerate case of the block layout: one scale per token (block_k = K)
# and one per output channel (block_n = 1), on the prefill shape
PER_CHANNEL = Linear("perchannel_int8_m4096_n14336_k4096", 4096, 14336, 4096, 0.015,
                     one_percent(4096), 30.0, INT8, 8, block_n=1, block_k=4096)
# the MXFP8 dense linear on the FP8 shape (1 x 32 scale groups on both sides)
MX_LINEAR = Linear("mxfp8_m2048_n4096_k14336", 2048, 4096, 14336, 0.01, 0, 1.0, MXFP8, 9,
                   block_n=1, block_k=32)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def activations(M: int, K: int, seed: int, n_outliers: int = 0, outlier_scale: float = 1.0,
                device="cpu") -> torch.Tensor:
    """bf16 [M, K]: N(0,1) with `n_outliers` whole channels multiplied by
    `outlier_scale`.  Channels are drawn by the same seed."""
    g = _gen(seed, device)
    x = torch.randn(M, K, generator=g, device=device, dtype=torch.float32)
    if n_outliers > 0:
        ch = torch.randperm(K, generator=g, device=device)[:n_outliers]
        x[:, ch] *= outlier_scale
    return x.to(torch.bfloat16)


def weights(N: int, K: int, std: float, seed: int, device="cpu", batch: int | None = None
            ) -> torch.Tensor:
    """fp32 [N, K] (or [batch, N, K]) ~ N(0, std^2)."""
    g = _gen(seed + 1000003, device)
    shape = (N, K) if batch is None else (batch, N, K)
    w = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    return w.mul_(std)


def linear_inputs(cfg: Linear, device="cpu"):
    """(A bf16 [M, K], W fp32 [N, K]) for a linear workload."""
    a = activations(cfg.M, cfg.K, cfg.seed, cfg.n_outliers, cfg.outlier_scale, device)
    w = weights(cfg.N, cfg.K, cfg.w_std, cfg.seed, device)
    return a, w


def router_logits(T: int, E: int, seed: int) -> torch.Tensor:
    """The router logits of the MoE workload: fp32 [T, E] ~ N(0, 1) (CPU)."""
    g = _gen(seed + 7919, "cpu")
    return torch.randn(T, E, generator=g, dtype=torch.float32)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bf16_bits(h: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(h, dtype=np.uint16).view(np.int16)).view(
        torch.bfloat16)


def cdiv(a: int, b: int) -> int:
    return -(-a // b)


