"""Seeded synthetic inputs for the five workloads.

This module holds no quantisation arithmetic: it only draws seeded random tensors (numpy PCG64)
and rounds them to the storage dtype (torch's round-to-nearest-even cast).  The CUDA tests, the
bench and the oracle all take their inputs from here, so both sides see identical bits.

Workloads (shapes are parameters so the same recipe serves small parity cases):
  mx_small      fp32 N(0,1)                                  seed 0      (256 x 512)
  nv_outliers   bf16 N(0,1), round(0.1% of cols) columns x U(50,100)   seed 5      (8192 x 8192)
  fwht_laplace  bf16 Laplace(0,1), 8 channels set to 120.0            seed 6      (16384 x 8192)
  gemm_normal   bf16 N(0,1)                                  seeds 1, 2  (8192 x 8192 each)
  swiglu_act    bf16 silu(g) * u, g, u ~ N(0,1)              seed 3      (4096 x 28672)
  weight        bf16 N(0, 0.02)                              seed 4      (8192 x 28672)
  lattice_steps k / 8 for integers k uniform in [-48, 48]       (parity cases: exact ties between
                                                                 the two four-over-six candidates)
  rht_signs     d fair sign bits, packed in uint32 words         (randomised rotation)
  swiglu_inputs bf16 g, u ~ N(0,1), streams (3,0) and (3,1)       (fused SwiGLU -> rotation path)
"""
from __future__ import annotations

import numpy as np
import torch


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def normal_f32(rows: int, cols: int, seed: int, std: float = 1.0) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return torch.from_numpy(x)


def normal_bf16(rows: int, cols: int, seed: int, std: float = 1.0) -> torch.Tensor:
    return normal_f32(rows, cols, seed, std).to(torch.bfloat16)


def mx_small(rows: int = 256, cols: int = 512, seed: int = 0) -> torch.Tensor:
    """fp32 N(0,1) activation for the MXFP4 quantise + dequantise case."""
    return normal_f32(rows, cols, seed)


def nv_outliers(rows: int = 8192, cols: int = 8192, seed: int = 5) -> torch.Tensor:
    """bf16 N(0,1) with round(0.1% of the columns) picked by a seeded permutation, each column
    multiplied by its own U(50, 100) factor (emergent outlier channels)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    n_out = max(1, int(round(0.001 * cols)))
    cols_out = rng.permutation(cols)[:n_out]
    factors = rng.uniform(50.0, 100.0, size=n_out).astype(np.float32)
    x[:, cols_out] *= factors[None, :]
    return _to_bf16(x)


def fwht_laplace(rows: int = 16384, d: int = 8192, seed: int = 6, n_spikes: int = 8,
                 spike: float = 120.0) -> torch.Tensor:
    """bf16 Laplace(0,1) tokens with `n_spikes` seeded channels set to `spike` in every token."""
    rng = np.random.default_rng(seed)
    mag = rng.standard_exponential((rows, d), dtype=np.float32)
    sign = rng.integers(0, 2, size=(rows, d), dtype=np.int8)
    x = np.where(sign == 1, mag, -mag)
    ch = rng.choice(d, size=n_spikes, replace=False)
    x[:, ch] = np.float32(spike)
    return _to_bf16(x)


def gemm_operand(rows: int, cols: int, seed: int) -> torch.Tensor:
    """bf16 N(0,1) GEMM operand (A uses seed 1, B seed 2)."""
    return normal_bf16(rows, cols, seed)


def swiglu_act(rows: int = 4096, cols: int = 28672, seed: int = 3) -> torch.Tensor:
    """bf16(silu(g) * u) with g, u ~ N(0,1) drawn from two streams of one seed."""
    g = np.random.default_rng([seed, 0]).standard_normal((rows, cols), dtype=np.float32)
    u = np.random.default_rng([seed, 1]).standard_normal((rows, cols), dtype=np.float32)
    a = g / (np.float32(1.0) + np.exp(-g)) * u
    return _to_bf16(a)


def swiglu_inputs(rows: int, cols: int, seed: int = 3) -> tuple[torch.Tensor, torch.Tensor]:
    """The two bf16 inputs g, u ~ N(0,1) of the fused SwiGLU path, from the same two streams as
    swiglu_act (each rounded to bf16; the activation itself is formed by the path under test)."""
    g = np.random.default_rng([seed, 0]).standard_normal((rows, cols), dtype=np.float32)
    u = np.random.default_rng([seed, 1]).standard_normal((rows, cols), dtype=np.float32)
    return _to_bf16(g), _to_bf16(u)


def weight(rows: int = 8192, cols: int = 28672, seed: int = 4, std: float = 0.02) -> torch.Tensor:
    return normal_bf16(rows, cols, seed, std)


def lattice_steps(rows: int, cols: int, seed: int, denom: int = 8, kmax: int = 48) -> torch.Tensor:
    """bf16 values k / denom, k uniform on [-kmax, kmax] (exact in bf16).  Such blocks sit on or
    near both four-over-six grids at once, so many of them have equal or nearly equal block
    errors under the two candidates."""
    rng = np.random.default_rng(seed)
    k = rng.integers(-kmax, kmax + 1, size=(rows, cols))
    return _to_bf16((k / denom).astype(np.float32))


def rht_signs(d: int, seed: int) -> np.ndarray:
    """Sign vector of the randomised rotation: d independent fair bits, packed 32 per uint32 word
    (bit i % 32 of word i // 32 set = channel i negated)."""
    rng = np.random.default_rng(seed)
    return rng.integers(0, 2 ** 32, size=d // 32, dtype=np.uint64).astype(np.uint32)


def as_f32_numpy(t: torch.Tensor) -> np.ndarray:
    """Exact fp32 view of a CPU tensor (bf16 -> fp32 is exact)."""
    return t.float().contiguous().numpy()
