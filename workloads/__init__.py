"""Seeded synthetic inputs for the ConvRot256 INT8 linear path.

This module only draws random numbers. It holds none of the method's
arithmetic (no rotation, no quantisation, no GEMM), so both the CPU oracle
(``oracle/``) and the CUDA path (the package) can take their inputs from it
without sharing any code with each other.

The workloads stand in for the diffusion-transformer linears timed on the
sglang page "Tune Kitchen INT8 row splitting for SM120" (Benchmark & Profiling
table: H3 QKV projections such as M32700/K5376/N16128). Those models' weights
and activations are not available, so the inputs are synthetic:

1. ``X``: M x K fp32 draws, ``standard_normal`` (Laplace(0, 1) for the
   long-reduction case), then ``n_outlier`` distinct columns picked by
   ``rng.choice`` are multiplied by 20 (outlier channels, the reason a
   rotation is applied before per-row quantisation), then cast to BF16
   with round-to-nearest-even (torch's CPU cast).
2. ``W``: N x K fp32 ``standard_normal`` times ``w_std``.
3. ``bias``: N fp32 ``standard_normal`` times ``b_std``, cast to BF16.

The draws happen in exactly that order from ``numpy.random.default_rng(seed)``
(PCG64), so every consumer that asks for the same config gets the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class Config:
    name: str
    M: int
    K: int
    N: int
    seed: int
    x_dist: str  # "normal" or "laplace"
    n_outlier: int
    w_std: float
    b_std: float

    @property
    def ops(self) -> int:
        """2*M*N*K: the multiply-adds of the INT8 GEMM, counted as two ops."""
        return 2 * self.M * self.N * self.K


def _n_out(K: int) -> int:
    return math.ceil(0.005 * K)


CONFIGS = [
    Config("tiny_m128_k512_n512", 128, 512, 512, 0, "normal", 4, 0.02, 0.01),
    Config("ragged_m8193_k5376_n16128", 8193, 5376, 16128, 1, "normal", _n_out(5376), 0.02, 0.01),
    Config("qkv_m32700_k5376_n16128", 32700, 5376, 16128, 2, "normal", _n_out(5376), 0.02, 0.01),
    Config("mlp_up_m14850_k7168_n28672", 14850, 7168, 28672, 3, "normal", _n_out(7168), 0.02, 0.01),
    Config("mlp_down_m14850_k28672_n7168", 14850, 28672, 7168, 4, "laplace", _n_out(28672), 0.01, 0.01),
]

BY_NAME = {c.name: c for c in CONFIGS}

# The shape the headline throughput is quoted on (M32700/K5376/N16128).
HEADLINE = CONFIGS[2]


def custom(M: int, K: int, N: int, seed: int = 1234, x_dist: str = "normal",
           n_outlier: int | None = None, w_std: float = 0.02, b_std: float = 0.01) -> Config:
    """A config of any shape with the same distributions (for ragged/edge tests)."""
    if n_outlier is None:
        n_outlier = min(K, max(1, _n_out(K)))
    return Config(f"custom_m{M}_k{K}_n{N}_s{seed}", M, K, N, seed, x_dist, n_outlier, w_std, b_std)


def _draw_x(rng: np.random.Generator, cfg: Config) -> np.ndarray:
    if cfg.x_dist == "normal":
        return rng.standard_normal((cfg.M, cfg.K), dtype=np.float32)
    if cfg.x_dist == "laplace":
        return rng.laplace(0.0, 1.0, (cfg.M, cfg.K)).astype(np.float32)
    raise ValueError(f"unknown x_dist {cfg.x_dist!r}")


def make_inputs(cfg: Config):
    """Return (X bf16 [M,K], W fp32 [N,K], bias bf16 [N]) as CPU torch tensors."""
    rng = np.random.default_rng(cfg.seed)
    x = _draw_x(rng, cfg)
    if cfg.n_outlier > 0:
        cols = rng.choice(cfg.K, cfg.n_outlier, replace=False)
        x[:, cols] *= np.float32(20.0)
    w = rng.standard_normal((cfg.N, cfg.K), dtype=np.float32)
    w *= np.float32(cfg.w_std)
    b = rng.standard_normal(cfg.N, dtype=np.float32)
    b *= np.float32(cfg.b_std)
    X = torch.from_numpy(x).to(torch.bfloat16)
    del x
    W = torch.from_numpy(w)
    bias = torch.from_numpy(b).to(torch.bfloat16)
    return X, W, bias


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a CPU bf16 tensor as a numpy uint16 array of its bit patterns (no copy)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bf16_bits(a: np.ndarray) -> torch.Tensor:
    """Inverse of :func:`bf16_bits`."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
