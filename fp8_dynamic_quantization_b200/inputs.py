"""Seeded synthetic inputs for the five workloads of the FP8 linear path.

This module only draws random numbers and arranges them into tensors; it holds
none of the quantisation or GEMM arithmetic, so both the CUDA path and the CPU
oracle can take their inputs from it.

Every tensor is generated on the host with ``numpy.random.Generator(PCG64)``
in float64, rounded to float32 by numpy and then to bf16 (round-to-nearest-
even) by torch.  The seed of a shape is ``1000 * workload + index of the shape
in that workload's sweep`` unless the caller passes another.

Workloads (the shapes follow the pages' activations and projection sizes):

1. tiny linear layer: X[64,2048] ~ N(0,1) with 4 seed-chosen K-columns x50;
   W[2048,2048] ~ N(0,1).
2. per-tensor sweep: X[M,2048] ~ N(0,1), M in {1,64,256,1024,65536}; every
   16th row (rows 0, 16, 32, ...) scaled by U(1,100) drawn per row; one
   128-wide group of row M//2 (group index drawn from the seed) set to +0.
3. group-quant sweep: X[M,7168] ~ Laplace(0,1), M in {1,32,4096,16384};
   72 seed-chosen K-columns (1% of 7168) x100.
4. decode GEMM: E4M3 codes uniform over the 254 finite codes (0x7F and 0xFF
   excluded), A [M,7168], B [N,7168]; scales U(1e-3, 1e-1) fp32, sa [M,56],
   sb [ceil(N/128),56]; M in {1,16,64,256}, N in {2048,7168,18432}.
5. prefill path: X[4096,7168] ~ N(0,1) with 72 seed-chosen K-columns x50;
   B codes and scales drawn as in workload 4 for N in {7168,18432,24576}.
"""
from __future__ import annotations

import numpy as np
import torch

K_SMALL = 2048
K_LARGE = 7168

WORKLOAD_SHAPES = {
    1: [(64, 2048, 2048)],                                   # (M, N, K)
    2: [(m, 0, 2048) for m in (1, 64, 256, 1024, 65536)],
    3: [(m, 0, 7168) for m in (1, 32, 4096, 16384)],
    4: [(m, n, 7168) for m in (1, 16, 64, 256) for n in (2048, 7168, 18432)],
    5: [(4096, n, 7168) for n in (7168, 18432, 24576)],
}

# The 254 codes that encode finite values (0x7F / 0xFF are the NaN codes).
FINITE_E4M3_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F],
                             dtype=np.uint8)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def to_bf16(values: np.ndarray) -> torch.Tensor:
    """float64/float32 numpy array -> bf16 torch CPU tensor (RNE via fp32)."""
    f32 = np.ascontiguousarray(values, dtype=np.float32)
    return torch.from_numpy(f32).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The uint16 bit patterns of a CPU bf16 tensor (shares strides)."""
    return t.view(torch.int16).numpy().view(np.uint16)


def _outlier_columns(g: np.random.Generator, k: int, count: int) -> np.ndarray:
    return np.sort(g.choice(k, size=count, replace=False))


def activations_tiny(seed: int = 1000) -> torch.Tensor:
    """Workload 1 activation X[64,2048]."""
    g = rng(seed)
    x = g.standard_normal((64, K_SMALL))
    x[:, _outlier_columns(g, K_SMALL, 4)] *= 50.0
    return to_bf16(x)


def weight_tiny(seed: int = 1001) -> torch.Tensor:
    """Workload 1 weight W[2048,2048] ~ N(0,1)."""
    return to_bf16(rng(seed).standard_normal((K_SMALL, K_SMALL)))


def activations_per_tensor(m: int, seed: int | None = None,
                           k: int = K_SMALL) -> torch.Tensor:
    """Workload 2 activation X[m,k] with row outliers and one zero group."""
    if seed is None:
        sizes = [s[0] for s in WORKLOAD_SHAPES[2]]
        seed = 2000 + (sizes.index(m) if m in sizes else 99)
    g = rng(seed)
    x = g.standard_normal((m, k))
    rows = np.arange(0, m, 16)
    x[rows, :] *= g.uniform(1.0, 100.0, size=rows.size)[:, None]
    if k >= 128:
        grp = int(g.integers(0, k // 128))
        x[m // 2, 128 * grp:128 * grp + 128] = 0.0
    return to_bf16(x)


def activations_group(m: int, seed: int | None = None, k: int = K_LARGE,
                      outlier_scale: float = 100.0,
                      dist: str = "laplace") -> torch.Tensor:
    """Workload 3 (Laplace, x100) or workload 5 (normal, x50) activation."""
    if seed is None:
        sizes = [s[0] for s in WORKLOAD_SHAPES[3]]
        seed = 3000 + (sizes.index(m) if m in sizes else 99)
    g = rng(seed)
    if dist == "laplace":
        x = g.laplace(0.0, 1.0, size=(m, k))
    else:
        x = g.standard_normal((m, k))
    ncol = max(1, round(0.01 * k))
    x[:, _outlier_columns(g, k, ncol)] *= outlier_scale
    return to_bf16(x)


def activations_prefill(seed: int = 5000, m: int = 4096,
                        k: int = K_LARGE) -> torch.Tensor:
    """Workload 5 activation X[4096,7168] ~ N(0,1), 72 columns x50."""
    return activations_group(m, seed=seed, k=k, outlier_scale=50.0, dist="normal")


def e4m3_codes(g: np.random.Generator, shape) -> np.ndarray:
    """Codes drawn uniformly from the 254 finite E4M3 codes."""
    return FINITE_E4M3_CODES[g.integers(0, FINITE_E4M3_CODES.size, size=shape)]


def block_scales(g: np.random.Generator, shape) -> np.ndarray:
    return g.uniform(1e-3, 1e-1, size=shape).astype(np.float32)


def gemm_operands(m: int, n: int, k: int = K_LARGE, seed: int | None = None):
    """Workload 4 operands: (qa [m,k] u8, sa [m,k/128] f32,
    qb [n,k] u8, sb [ceil(n/128),k/128] f32) as numpy arrays."""
    if seed is None:
        shapes = WORKLOAD_SHAPES[4]
        seed = 4000 + (shapes.index((m, n, k)) if (m, n, k) in shapes else 99)
    g = rng(seed)
    G = k // 128
    qa = e4m3_codes(g, (m, k))
    sa = block_scales(g, (m, G))
    qb = e4m3_codes(g, (n, k))
    sb = block_scales(g, ((n + 127) // 128, G))
    return qa, sa, qb, sb


def weight_operands(n: int, k: int = K_LARGE, seed: int = 5100):
    """Workload 5 weight codes and scales: (qb [n,k] u8, sb [ceil(n/128),k/128])."""
    g = rng(seed + n)
    return e4m3_codes(g, (n, k)), block_scales(g, ((n + 127) // 128, k // 128))
