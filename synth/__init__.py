"""Seeded synthetic inputs shared by the oracle checks and the CUDA path.

This module only draws random numbers and lays them out; it holds none of the
quantized-linear arithmetic.  Every tensor comes from numpy's PCG64 generator
seeded per workload, so the oracle and the GPU see identical bytes.

bf16 tensors are returned as uint16 bit patterns (numpy has no bf16 dtype):
fp32 draws rounded to the nearest bf16, ties to even.  fp16 scales are numpy
float16 values (also round-to-nearest-even from the fp32 draw).

Workloads (sizes and distributions of the quantized-linear benchmark set):
  bitlinear_tiny     x fp32 [8,256] ~N(0,1); W fp32 [128,256] ~N(0,0.02)
  gemm_w8a8          x, w int8 [4096,4096] uniform in [-128,127];
                     deqScale, perTokenScale fp32 [4096] ~U(0.001,0.01)
  bitlinear_decode   x bf16 [M,4096] ~N(0,1), M in {1,4,16};
                     W fp32 [11008,4096] ~N(0,0.02)
  linear_w4_grouped  codes uint8 [14336,4096] uniform 0..15; fp16 scales
                     [14336,32] ~U(0.005,0.02); zero-points uint8 [14336,32]
                     uniform 0..15; bias fp32 [14336] ~N(0,0.01);
                     x fp32 [M,4096] ~N(0,1), M in {1,32}
  bitlinear_prefill  x bf16 [8192,4096] ~N(0,1), 41 outlier channels (1% of
                     K, a seeded permutation) each scaled by 1+|N(0,3)|;
                     W fp32 [4096,4096] ~N(0,0.02)
"""
from __future__ import annotations

import numpy as np


def rng(seed) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_f32(g: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = g.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def uniform_f32(g: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    return g.uniform(lo, hi, shape).astype(np.float32)


def int8_uniform(g: np.random.Generator, shape) -> np.ndarray:
    return g.integers(-128, 128, shape, dtype=np.int16).astype(np.int8)


def nibbles(g: np.random.Generator, shape) -> np.ndarray:
    return g.integers(0, 16, shape, dtype=np.uint8)


# --------------------------------------------------------------------------
# Named workloads
# --------------------------------------------------------------------------

def bitlinear_tiny(seed: int = 0):
    g = rng(seed)
    x = normal_f32(g, (8, 256))
    w = normal_f32(g, (128, 256), 0.02)
    return {"x": x, "w": w, "eps": 1e-5}


def gemm_w8a8(M: int = 4096, N: int = 4096, K: int = 4096, seed: int = 2):
    g = rng(seed)
    x = int8_uniform(g, (M, K))
    w = int8_uniform(g, (N, K))
    deq = uniform_f32(g, (N,), 0.001, 0.01)
    pts = uniform_f32(g, (M,), 0.001, 0.01)
    return {"x": x, "w": w, "deq_scale": deq, "per_token_scale": pts}


def bitlinear_weight(N: int, K: int, seed: int, std: float = 0.02):
    return normal_f32(rng(seed), (N, K), std)


def bf16_activations(M: int, K: int, seed, outlier_frac: float = 0.0):
    """x ~N(0,1) (optionally with outlier channels), as bf16 bits and exact fp32."""
    g = rng(seed)
    x = normal_f32(g, (M, K))
    if outlier_frac > 0.0:
        n_out = int(round(outlier_frac * K))
        ch = g.permutation(K)[:n_out]
        mult = (1.0 + np.abs(g.normal(0.0, 3.0, n_out))).astype(np.float32)
        x[:, ch] *= mult[None, :]
    bits = f32_to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits)


def bitlinear_decode(M: int, N: int = 11008, K: int = 4096, seed: int = 3):
    bits, xf = bf16_activations(M, K, (seed, M))
    w = bitlinear_weight(N, K, seed)
    return {"x_bf16": bits, "x": xf, "w": w, "eps": 1e-5}


def bitlinear_prefill(M: int = 8192, N: int = 4096, K: int = 4096, seed: int = 5):
    bits, xf = bf16_activations(M, K, (seed, 0), outlier_frac=0.01)
    w = bitlinear_weight(N, K, seed)
    return {"x_bf16": bits, "x": xf, "w": w, "eps": 1e-5}


def linear_w4_weights(N: int = 14336, K: int = 4096, group_size: int = 128, seed: int = 4):
    g = rng(seed)
    G = K // group_size
    q = nibbles(g, (N, K))
    scales = g.uniform(0.005, 0.02, (N, G)).astype(np.float16)
    zeros = nibbles(g, (N, G))
    bias = normal_f32(g, (N,), 0.01)
    return {"q": q, "scales_f16": scales, "zeros": zeros, "bias": bias, "group_size": group_size}


def linear_w4_activations(M: int, K: int = 4096, seed: int = 4):
    return normal_f32(rng((seed, M)), (M, K))
