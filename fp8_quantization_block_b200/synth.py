"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds no quantization or GEMM arithmetic: it only draws random
numbers and rounds them to bf16, so that the CUDA path and the CPU oracle can
be fed the very same bytes.  All draws use numpy's PCG64 with an explicit
seed; values are drawn in fp64, cast to fp32 and rounded to bf16 with
round-to-nearest-even (torch's cast).

Workloads (sizes follow the diffusion-transformer and LLM Linear layers the
pages discuss; no model or dataset is used):

* ``tiny_pair``       A, B [64 x 256], N(0, 1), 1% of entries x50, seed 0
                      (A drawn first, then B from the same generator).
* ``dit_activations`` X [4096 x 3072], N(0, 1), 8 outlier channels x30
                      (the first 8 of a seeded permutation of the K columns).
* ``gaussian_weights`` W [N x K], N(0, 0.02^2).
* ``student_t``       X ~ t(nu = 3) drawn as Z / sqrt(chi2_3 / 3), chi2_3 the
                      sum of 3 squared normals from the same generator.
* ``sweep_tensor``    [M x 4096], N(0, 1), 0.5% of entries x100.
"""
from __future__ import annotations

import numpy as np
import torch


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32/fp64 numpy array -> bf16 bit patterns (uint16), RNE."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_tensor(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> torch.bfloat16 CPU tensor (same bytes)."""
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_with_outliers(rng: np.random.Generator, shape, p: float, factor: float) -> np.ndarray:
    x = rng.standard_normal(shape)
    mask = rng.random(shape) < p
    return np.where(mask, x * factor, x)


def tiny_pair(seed: int = 0, M: int = 64, N: int = 64, K: int = 256):
    rng = _rng(seed)
    A = normal_with_outliers(rng, (M, K), 0.01, 50.0)
    B = normal_with_outliers(rng, (N, K), 0.01, 50.0)
    return to_bf16_bits(A), to_bf16_bits(B)


def dit_activations(seed: int = 1, M: int = 4096, K: int = 3072, n_outlier: int = 8,
                    factor: float = 30.0) -> np.ndarray:
    rng = _rng(seed)
    x = rng.standard_normal((M, K))
    cols = rng.permutation(K)[:n_outlier]
    x[:, cols] *= factor
    return to_bf16_bits(x)


def gaussian_weights(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    rng = _rng(seed)
    return to_bf16_bits(rng.standard_normal((N, K)) * std)


def student_t(seed: int, M: int, K: int, nu: int = 3) -> np.ndarray:
    rng = _rng(seed)
    z = rng.standard_normal((M, K))
    chi2 = np.zeros((M, K))
    for _ in range(nu):
        chi2 += rng.standard_normal((M, K)) ** 2
    return to_bf16_bits(z / np.sqrt(chi2 / nu))


def kv_cache(seed: int, tokens: int, layers: int = 80, kv_heads: int = 8, head_dim: int = 128,
             outlier_dims: int = 2, factor: float = 15.0) -> np.ndarray:
    """K/V cache entries of a grouped-query-attention model: one row per
    (token, layer, K or V), row = kv_heads * head_dim values (heads
    contiguous, each head_dim contiguous).  N(0, 1); in the K rows, a seeded
    set of `outlier_dims` dimensions per head and layer is scaled by `factor`
    (keys carry fixed outlier channels, values do not)."""
    rng = _rng(seed)
    x = rng.standard_normal((tokens, layers, 2, kv_heads, head_dim))
    for layer in range(layers):
        for h in range(kv_heads):
            dims = rng.permutation(head_dim)[:outlier_dims]
            x[:, layer, 0, h, dims] *= factor
    return to_bf16_bits(x.reshape(tokens * layers * 2, kv_heads * head_dim))


def sweep_tensor(seed: int, M: int, K: int = 4096) -> np.ndarray:
    rng = _rng(seed)
    return to_bf16_bits(normal_with_outliers(rng, (M, K), 0.005, 100.0))


def edge_rows(K: int) -> np.ndarray:
    """Hand-built rows that exercise the corners of the codecs: zeros, -0,
    bf16 subnormals, the largest bf16, exact powers of two, and a mix."""
    rows = []
    rows.append(np.zeros(K, dtype=np.float32))
    rows.append(-np.zeros(K, dtype=np.float32))
    sub = np.float32(2.0 ** -130)
    rows.append(np.full(K, sub, dtype=np.float32) * np.where(np.arange(K) % 2 == 0, 1, -1))
    big = np.float32(3.3895314e38)
    rows.append(np.where(np.arange(K) % 3 == 0, big, -big / 3).astype(np.float32))
    rows.append((2.0 ** ((np.arange(K) % 40) - 20)).astype(np.float32))
    rows.append(np.linspace(-7.0, 7.0, K).astype(np.float32))
    mix = np.zeros(K, dtype=np.float32)
    mix[::7] = 1e-3
    mix[::11] = -5.5
    rows.append(mix)
    return to_bf16_bits(np.stack(rows))


def tie_rows(K: int, fmt: int) -> np.ndarray:
    """Rows whose block maximum pins the scale so that other elements land
    exactly on E2M1 / E4M3 / E5M2 / E3M2 rounding midpoints (MX formats:
    scale = 1)."""
    if fmt in (2, 3):
        mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 5.5, 6.5, 0.125, 0.375]
        top = 6.0
    elif fmt == 0:
        mids = [1.0625, 1.1875, 17.0, 19.0, 240.0, 416.0, 432.0, 2.0 ** -10, 3 * 2.0 ** -10]
        top = 448.0
    elif fmt == 4:   # E3M2
        mids = [2.0 ** -5, 3 * 2.0 ** -5, 0.28125, 1.125, 1.375, 2.25, 3.75, 4.5, 6.5, 7.5, 9.0, 13.0, 15.0, 18.0, 26.0]
        top = 28.0
    else:
        mids = [1.125, 1.375, 2.5, 3.5, 40960.0, 2.0 ** -17, 3 * 2.0 ** -17]
        top = 57344.0
    bs = 16 if fmt == 3 else 32
    row = np.zeros(K, dtype=np.float32)
    for b in range(K // bs):
        blk = np.array([(-1) ** (i + b) * mids[(i + b) % len(mids)] for i in range(bs)], dtype=np.float32)
        blk[0] = top
        row[b * bs:(b + 1) * bs] = blk
    return to_bf16_bits(np.stack([row, -row]))
