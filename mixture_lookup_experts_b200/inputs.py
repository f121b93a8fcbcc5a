"""Seeded synthetic inputs for the MoLE lookup path (host side, numpy).

This module draws random numbers and nothing else: it holds none of the
method's arithmetic, so both the CUDA path and the CPU oracle can be fed from
it.  Shapes follow the model sizes the MoLE page trains ("ICML 2025 Spotlight |
华为诺亚提出端侧大模型新架构MoLE...", section 实验结果: 160M / 410M / 1B activated
parameters, expert width equal to the dense FFN).  The page's training data (a
100B-token Pile subset) is not available; these draws stand in for it.

Recipe (one numpy ``default_rng(seed)`` per config, tensors drawn in the fixed
order E, W1, W2, Wr, ids, h):
  E, W1, W2, Wr ~ N(0, 0.02);  h ~ N(0, 1)
  ids: Zipf(s=1.1) over the vocabulary (P(rank k) ~ k^-1.1, rank k -> id k-1,
       sampled by inverse CDF) or uniform over [0, V).
bf16 tensors are returned as uint16 bit patterns (fp32 draw rounded to
nearest-even), fp32 tensors as float32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Shape:
    name: str
    V: int
    D: int
    N: int
    Dr: int
    layers: int
    dtype: str          # "f32" or "bf16"
    tokens: tuple = field(default=())
    seed: int = 0


# The five workloads: a tiny fp32 layer and the 160M / 410M / 1B-activated
# shaped layers (bf16 table), the last also as an NF3-compressed table.
SHAPES = {
    "tiny": Shape("tiny", V=512, D=64, N=4, Dr=256, layers=1, dtype="f32", tokens=(256,), seed=1001),
    "160m": Shape("160m", V=50304, D=768, N=16, Dr=3072, layers=12, dtype="bf16", tokens=(1, 8, 64), seed=1002),
    "410m": Shape("410m", V=50304, D=1024, N=16, Dr=4096, layers=24, dtype="bf16",
                  tokens=(1, 2, 4, 8, 16, 32, 64, 128, 256), seed=1003),
    "1b": Shape("1b", V=50304, D=2048, N=16, Dr=8192, layers=16, dtype="bf16", tokens=(4096, 16384), seed=1004),
    "1b_nf3": Shape("1b_nf3", V=50304, D=2048, N=16, Dr=8192, layers=16, dtype="bf16",
                    tokens=(1, 8, 64, 256, 1024, 4096, 16384), seed=1005),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    x = (rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)).astype(np.float32)
    return f32_to_bf16_bits(x) if dtype == "bf16" else x


def zipf_ids(rng: np.random.Generator, T: int, V: int, s: float = 1.1) -> np.ndarray:
    """T ids with P(id = k-1) proportional to k^-s, k = 1..V (inverse CDF)."""
    k = np.arange(1, V + 1, dtype=np.float64)
    cdf = np.cumsum(k ** (-s))
    cdf /= cdf[-1]
    u = rng.random(T)
    return np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int32)


def uniform_ids(rng: np.random.Generator, T: int, V: int) -> np.ndarray:
    return rng.integers(0, V, size=T, dtype=np.int64).astype(np.int32)


def draw_ids(rng: np.random.Generator, T: int, V: int, kind: str) -> np.ndarray:
    if kind == "zipf":
        return zipf_ids(rng, T, V)
    if kind == "uniform":
        return uniform_ids(rng, T, V)
    raise ValueError(kind)


def expert_weights(shape: Shape, seed: int | None = None, std: float = 0.02):
    """E [V, D], W1 [N, D, Dr], W2 [N, Dr, D] in the shape's dtype."""
    rng = np.random.default_rng(shape.seed if seed is None else seed)
    E = normal(rng, (shape.V, shape.D), std, shape.dtype)
    W1 = normal(rng, (shape.N, shape.D, shape.Dr), std, shape.dtype)
    W2 = normal(rng, (shape.N, shape.Dr, shape.D), std, shape.dtype)
    return rng, E, W1, W2


def router_and_batch(rng: np.random.Generator, shape: Shape, T: int, ids_kind: str = "uniform",
                     std: float = 0.02):
    """Wr [D, N], ids [T], h [T, D] drawn after the expert weights."""
    Wr = normal(rng, (shape.D, shape.N), std, shape.dtype)
    ids = draw_ids(rng, T, shape.V, ids_kind)
    h = normal(rng, (T, shape.D), 1.0, shape.dtype)
    return Wr, ids, h


def small(V: int, D: int, N: int, Dr: int, dtype: str, seed: int, std: float = 0.02) -> Shape:
    """An ad-hoc shape for parity tests at oracle-friendly sizes."""
    return Shape(f"v{V}d{D}n{N}r{Dr}{dtype}", V=V, D=D, N=N, Dr=Dr, layers=1, dtype=dtype, seed=seed)


def expected_unique_zipf(T: int, V: int, s: float = 1.1) -> float:
    """E[#distinct ids] among T Zipf(s) draws: sum_k 1 - (1 - p_k)^T."""
    k = np.arange(1, V + 1, dtype=np.float64)
    p = k ** (-s)
    p /= p.sum()
    return float(np.sum(1.0 - np.exp(T * np.log1p(-p))))
