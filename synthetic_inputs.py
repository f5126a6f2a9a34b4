"""Seeded synthetic inputs for the W4A8 GEMM workloads.

This module only draws random numbers and holds the workload shapes; it
contains none of the method's arithmetic.  Both the oracle-side tests and the
CUDA-side tests/benchmark use it, so the two sides see identical inputs.

Recipe (all draws from ``numpy.random.default_rng(seed)``, PCG64):

* weights ``W`` (N x K, the [out, in] layout of a linear layer):
  ``standard_normal(float32) * sigma`` cast to float16, then a set of output
  rows chosen with ``choice(N, count, replace=False)`` scaled by a factor;
* activations ``X`` (M x K): ``standard_normal(float32)`` cast to float16,
  then a set of input channels (columns) chosen the same way, scaled;
* the pure-throughput sweep draws the quantized operands directly:
  codes q ~ U{0..15}, zeros z ~ U{0..15}, group scales s2 ~ U{1..8},
  per-channel / per-token scales ~ U[0.5, 1.5] * 1e-3 (float16) and
  activations X8 ~ U{-127..127}.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Layer:
    """One linear layer shape of a named model (shapes only, no weights)."""
    name: str
    K: int
    N: int
    group: int
    ms: tuple
    w_sigma: float
    x_outlier_frac: float
    x_outlier_scale: float
    w_outlier_rows: int = 0
    w_outlier_scale: float = 1.0
    x_outlier_count: int | None = None


# Small case the oracle finishes in seconds (parity workload).
TINY = Layer("tiny_w4a8", K=512, N=512, group=128, ms=(16,), w_sigma=0.02,
             x_outlier_frac=0.0, x_outlier_scale=20.0, w_outlier_rows=4,
             w_outlier_scale=8.0, x_outlier_count=2)

# Llama-3-8B fused QKV projection (32 query heads + 8 kv heads, head dim 128).
LLAMA3_8B_QKV = Layer("llama3_8b_qkv", K=4096, N=6144, group=128,
                      ms=(1, 16, 64, 256, 1024, 4096), w_sigma=0.02,
                      x_outlier_frac=0.01, x_outlier_scale=20.0)

LLAMA3_8B_GATE_UP = Layer("llama3_8b_gate_up", K=4096, N=28672, group=128,
                          ms=(1, 8, 32, 128, 512, 2048), w_sigma=0.02,
                          x_outlier_frac=0.01, x_outlier_scale=20.0)

LLAMA3_8B_DOWN = Layer("llama3_8b_down", K=14336, N=4096, group=128,
                       ms=(1, 8, 32, 128, 512, 2048), w_sigma=0.02,
                       x_outlier_frac=0.01, x_outlier_scale=20.0)

QWEN15_72B_QKV = Layer("qwen1.5_72b_qkv", K=8192, N=24576, group=128,
                       ms=(1, 16, 64, 256, 1024), w_sigma=0.015,
                       x_outlier_frac=0.005, x_outlier_scale=30.0)

QWEN15_72B_GATE_UP = Layer("qwen1.5_72b_gate_up", K=8192, N=49152, group=128,
                           ms=(1, 16, 64, 256, 1024), w_sigma=0.015,
                           x_outlier_frac=0.005, x_outlier_scale=30.0)

QWEN15_72B_DOWN = Layer("qwen1.5_72b_down", K=24576, N=8192, group=128,
                        ms=(1, 16, 64, 256, 1024), w_sigma=0.015,
                        x_outlier_frac=0.005, x_outlier_scale=30.0)

LAYERS = {l.name: l for l in (TINY, LLAMA3_8B_QKV, LLAMA3_8B_GATE_UP,
                              LLAMA3_8B_DOWN, QWEN15_72B_QKV,
                              QWEN15_72B_GATE_UP, QWEN15_72B_DOWN)}

# Shape sweep for the roofline crossover (random quantized operands).
SWEEP_KN = (2048, 4096, 8192)
SWEEP_MS = tuple(2 ** i for i in range(14))   # 1 .. 8192
SWEEP_GROUPS = (64, 128)


def _outlier_count(frac: float, dim: int) -> int:
    return int(round(frac * dim))


def weights(layer: Layer, seed: int = 0) -> np.ndarray:
    """W (N, K) float16, ~N(0, sigma) with optional scaled output rows."""
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((layer.N, layer.K), dtype=np.float32)
         * np.float32(layer.w_sigma)).astype(np.float16)
    if layer.w_outlier_rows:
        rows = rng.choice(layer.N, layer.w_outlier_rows, replace=False)
        W[rows] = (W[rows].astype(np.float32)
                   * np.float32(layer.w_outlier_scale)).astype(np.float16)
    return W


def activations(layer: Layer, M: int, seed: int = 0) -> np.ndarray:
    """X (M, K) float16, ~N(0, 1) with a few input channels scaled."""
    rng = np.random.default_rng(seed + 1_000_003 * (M + 1))
    X = rng.standard_normal((M, layer.K), dtype=np.float32).astype(np.float16)
    count = (layer.x_outlier_count if layer.x_outlier_count is not None
             else _outlier_count(layer.x_outlier_frac, layer.K))
    if count:
        cols = rng.choice(layer.K, count, replace=False)
        X[:, cols] = (X[:, cols].astype(np.float32)
                      * np.float32(layer.x_outlier_scale)).astype(np.float16)
    return X


def random_fp16(shape, seed: int, lo: float = -4.0, hi: float = 4.0):
    """Uniform float16 values (edge-case tests)."""
    rng = np.random.default_rng(seed)
    return rng.uniform(lo, hi, size=shape).astype(np.float32).astype(np.float16)


@dataclass
class SweepOperands:
    q: np.ndarray        # uint8 (N, K) codes 0..15
    s2: np.ndarray       # int8  (N, K/G) 1..8
    z: np.ndarray        # uint8 (N, K/G) 0..15
    s1: np.ndarray       # float16 (N,)
    X8: np.ndarray       # int8 (M, K)
    sx: np.ndarray       # float16 (M,)
    group: int = 128
    extra: dict = field(default_factory=dict)


def sweep_operands(M: int, N: int, K: int, group: int, seed: int = 0,
                   s2_max: int = 8) -> SweepOperands:
    """Quantized operands drawn directly (pure-throughput sweep)."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    z = rng.integers(0, 16, size=(N, K // group), dtype=np.uint8)
    s2 = rng.integers(1, s2_max + 1, size=(N, K // group), dtype=np.int8)
    s1 = (rng.uniform(0.5, 1.5, size=N) * 1e-3).astype(np.float16)
    X8 = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    sx = (rng.uniform(0.5, 1.5, size=M) * 1e-3).astype(np.float16)
    return SweepOperands(q=q, s2=s2, z=z, s1=s1, X8=X8, sx=sx, group=group)
