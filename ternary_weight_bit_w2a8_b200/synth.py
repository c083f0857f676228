"""Seeded synthetic inputs for the W2A8 BitLinear path.

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle. It only draws random numbers and encodes them (float32 -> bf16 bit
patterns); it holds none of the method's arithmetic: no ternarisation, no
activation quantisation, no packing and no contraction.

Workloads follow the shapes of the W2A8 GEMV benchmark page ("如何编译 BitNet
W2A8 CUDA 内核并用 test.py 运行 GEMV 加速测试？", section "运行 test.py 做 GEMV
基准测试": random int8 activations against ternary weights over eight (N, K)
shapes, plus the two extra kernel shapes listed under "限制与注意事项").
Every generator takes an explicit seed and uses numpy's PCG64
(``numpy.random.default_rng``); the order of draws is part of the recipe and is
stated in each docstring.
"""
from __future__ import annotations

import numpy as np

# (N, K) shapes of the GEMV shape sweep and of the two large kernel shapes.
SWEEP_SHAPES = [
    (2560, 2560), (3840, 2560), (13824, 2560), (2560, 6912),
    (3200, 3200), (4800, 3200), (3200, 10240), (20480, 3200),
]
LARGE_SHAPES = [(5120, 27648), (55296, 5120)]
BITLINEAR_DECODE_SHAPES = [(6912, 2560), (2560, 6912)]
PREFILL_M = [128, 512, 2048]
PREFILL_SHAPES = [(13824, 2560), (2560, 6912)]


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Encode float32 values as bf16 bit patterns (uint16), round to nearest even.

    Input encoding only. NaN is not produced by any generator here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def uniform_int8_ternary(N: int, K: int, seed: int = 0, M: int = 1):
    """Uniform int8 activations and equiprobable ternary weights.

    Draw order: q ~ integers[-127, 127] of shape (M, K), then W_t ~ integers
    [-1, 1] of shape (N, K) (P(-1) = P(0) = P(1) = 1/3).
    Returns (q int8 [M, K], W_t int8 [N, K]).
    """
    rng = np.random.default_rng(seed)
    q = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    w = rng.integers(-1, 2, size=(N, K), dtype=np.int8)
    return q, w


def sparse_ternary_normal_int8(N: int, K: int, seed: int = 0, M: int = 1,
                               p_zero: float = 0.4, sigma: float = 32.0):
    """Ternary weights with 40% zeros (+-1 split evenly) and N(0, 32) int8 activations.

    Draw order: u ~ uniform[0, 1) float32 of shape (N, K) gives
    W_t = -1 if u < (1-p_zero)/2, +1 if u >= (1+p_zero)/2, else 0; then
    g ~ N(0, sigma) of shape (M, K) gives q = rint(clip(g, -127, 127)).
    Returns (q int8 [M, K], W_t int8 [N, K]).
    """
    rng = np.random.default_rng(seed)
    u = rng.random(size=(N, K), dtype=np.float32)
    lo = np.float32((1.0 - p_zero) / 2.0)
    hi = np.float32((1.0 + p_zero) / 2.0)
    w = (u >= lo).astype(np.int8)
    w += (u >= hi).astype(np.int8)
    w -= 1
    del u
    g = rng.normal(0.0, sigma, size=(M, K))
    q = np.rint(np.clip(g, -127, 127)).astype(np.int8)
    return q, w


def bf16_activations(M: int, K: int, seed: int = 0, outlier_p: float = 0.01,
                     outlier_scale: float = 20.0) -> np.ndarray:
    """bf16 activations ~ N(0, 1), with an iid Bernoulli(outlier_p) mask scaled by outlier_scale.

    Draw order: g ~ N(0, 1) float64 of shape (M, K); then (only when
    outlier_p > 0) b ~ uniform[0, 1) of shape (M, K), and g is multiplied by
    outlier_scale where b < outlier_p. Returned as bf16 bit patterns
    (uint16 [M, K]).
    """
    rng = np.random.default_rng(seed)
    g = rng.normal(0.0, 1.0, size=(M, K))
    if outlier_p > 0.0:
        b = rng.random(size=(M, K))
        g = np.where(b < outlier_p, g * outlier_scale, g)
    return f32_to_bf16_bits(g.astype(np.float32))


def bf16_weights(N: int, K: int, seed: int = 0, sigma: float = 0.02) -> np.ndarray:
    """bf16 latent weights ~ N(0, sigma), as bf16 bit patterns (uint16 [N, K])."""
    rng = np.random.default_rng(seed)
    g = rng.normal(0.0, sigma, size=(N, K)).astype(np.float32)
    return f32_to_bf16_bits(g)


def bitlinear_inputs(M: int, N: int, K: int, seed: int = 0, outliers: bool = True):
    """Inputs for a full BitLinear call: (x bf16 bits [M, K], W bf16 bits [N, K]).

    x uses ``seed`` and W uses ``seed + 1``, each through its own generator, so
    a shape's weights do not depend on M.
    """
    x = bf16_activations(M, K, seed=seed, outlier_p=0.01 if outliers else 0.0)
    w = bf16_weights(N, K, seed=seed + 1)
    return x, w
