"""Seeded synthetic inputs for the W4A8 per-channel linear layer.

This module only draws numbers. It holds none of the quantization arithmetic,
so both the CPU oracle and the CUDA path can be fed from it without sharing
any of the method's code.

Workloads follow the shapes and value distributions of the pages' examples:

* the minimal Keras model of "INT4 quantization in Keras", section "Quantize a
  minimal functional model": inputs of shape 32x10 drawn uniformly from [0, 1),
  a Dense 10->32 layer with ReLU and a Dense 32->1 layer. Keras initialises a
  Dense kernel glorot-uniform and its bias to zero; the page's generator is
  unseeded, so we use our own seeded stream.
* decode / prefill / Gemma3-1B / 70B-shaped linears: weights N(0, sigma),
  activations N(0, 1) with a few "outlier" input channels scaled up, the data
  property described on the "4-bit-integer" concept page, section 3
  ("why LLM quantization is hard", point 1: emergent outlier channels).

Every array is float32, C-contiguous, laid out as the library expects:
weights W[K][N] (Keras kernel layout: rows = input features, columns = output
channels) and activations X[M][K] (rows = tokens).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# Sub-stream ids so that X, W and the outlier choice never share a stream.
_STREAM_X = 1
_STREAM_W = 2
_STREAM_OUTLIER = 3
_STREAM_BIAS = 4


def rng_for(seed: int, stream: int, sub: int = 0) -> np.random.Generator:
    """A numpy PCG64 generator keyed by (seed, stream, sub)."""
    return np.random.Generator(np.random.PCG64([int(seed), int(stream), int(sub)]))


def uniform01(shape, rng: np.random.Generator) -> np.ndarray:
    return rng.random(shape, dtype=np.float32)


def normal(shape, std: float, rng: np.random.Generator) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def glorot_uniform(fan_in: int, fan_out: int, rng: np.random.Generator) -> np.ndarray:
    """Keras' default Dense kernel initialiser: U(-l, l), l = sqrt(6 / (fan_in + fan_out))."""
    limit = math.sqrt(6.0 / (fan_in + fan_out))
    w = rng.uniform(-limit, limit, size=(fan_in, fan_out))
    return w.astype(np.float32)


def with_outlier_channels(x: np.ndarray, count: int, factor: float,
                          rng: np.random.Generator) -> tuple[np.ndarray, np.ndarray]:
    """Scale `count` input channels (columns of X[M][K]) by `factor` for every row.

    The channels are drawn without replacement. Returns (X, channel indices).
    """
    k = x.shape[1]
    idx = np.sort(rng.choice(k, size=min(count, k), replace=False))
    if idx.size:
        x[:, idx] *= np.float32(factor)
    return x, idx


# --------------------------------------------------------------------------
# Named workloads. Each returns plain float32 arrays; seeds are fixed per
# workload so the oracle and the kernels always see the same numbers.
# --------------------------------------------------------------------------

@dataclass
class MinimalMLP:
    x: np.ndarray        # [32][10]
    w1: np.ndarray       # [10][32]
    b1: np.ndarray       # [32]
    w2: np.ndarray       # [32][1]
    b2: np.ndarray       # [1]


def minimal_mlp(seed: int = 0) -> MinimalMLP:
    """Inputs 32x10 U[0,1); Dense 10->32 (ReLU) and Dense 32->1; glorot-uniform kernels, zero bias."""
    x = uniform01((32, 10), rng_for(seed, _STREAM_X))
    w1 = glorot_uniform(10, 32, rng_for(seed, _STREAM_W, 1))
    w2 = glorot_uniform(32, 1, rng_for(seed, _STREAM_W, 2))
    return MinimalMLP(x=x, w1=w1, b1=np.zeros(32, np.float32),
                      w2=w2, b2=np.zeros(1, np.float32))


@dataclass
class LinearCase:
    name: str
    x: np.ndarray | None        # [M][K] (None when only weights are asked for)
    w: np.ndarray               # [K][N]
    outliers: np.ndarray = field(default_factory=lambda: np.zeros(0, np.int64))


def linear_weights(k: int, n: int, std: float, seed: int, sub: int = 0) -> np.ndarray:
    return normal((k, n), std, rng_for(seed, _STREAM_W, sub))


def linear_activations(m: int, k: int, seed: int, sub: int = 0,
                       outlier_count: int = 0, outlier_factor: float = 1.0
                       ) -> tuple[np.ndarray, np.ndarray]:
    x = normal((m, k), 1.0, rng_for(seed, _STREAM_X, sub))
    idx = np.zeros(0, np.int64)
    if outlier_count:
        x, idx = with_outlier_channels(x, outlier_count, outlier_factor,
                                       rng_for(seed, _STREAM_OUTLIER, sub))
    return x, idx


def bias_vector(n: int, seed: int, sub: int = 0, std: float = 0.1) -> np.ndarray:
    return normal((n,), std, rng_for(seed, _STREAM_BIAS, sub))


# Decode single linear: K = N = 4096, M in {1, 4, 16}; W ~ N(0, 0.02);
# X ~ N(0, 1) with 8 random input channels x20.
DECODE_K = 4096
DECODE_N = 4096
DECODE_MS = (1, 4, 16)


def decode_case(m: int, seed: int = 1) -> LinearCase:
    w = linear_weights(DECODE_K, DECODE_N, 0.02, seed)
    x, idx = linear_activations(m, DECODE_K, seed, sub=m, outlier_count=8, outlier_factor=20.0)
    return LinearCase(f"decode_m{m}_k{DECODE_K}_n{DECODE_N}", x, w, idx)


# Prefill single linear: M = 2048, K = 4096, N = 11008; 0.5% of channels x20.
PREFILL_M, PREFILL_K, PREFILL_N = 2048, 4096, 11008


def prefill_case(seed: int = 2, m: int = PREFILL_M, k: int = PREFILL_K,
                 n: int = PREFILL_N) -> LinearCase:
    w = linear_weights(k, n, 0.02, seed)
    x, idx = linear_activations(m, k, seed, outlier_count=round(0.005 * k), outlier_factor=20.0)
    return LinearCase(f"prefill_m{m}_k{k}_n{n}", x, w, idx)


# Gemma3-1B-shaped stack: 26 layers x 7 projections, (K, N) each.
GEMMA_LAYERS = 26
GEMMA_PROJ = (("q", 1152, 1024), ("k", 1152, 256), ("v", 1152, 256), ("o", 1024, 1152),
              ("gate", 1152, 6912), ("up", 1152, 6912), ("down", 6912, 1152))
GEMMA_MS = (1, 512)


def gemma_weights(layer: int, proj: int, seed: int = 3) -> np.ndarray:
    _, k, n = GEMMA_PROJ[proj]
    return linear_weights(k, n, 0.02, seed, sub=layer * len(GEMMA_PROJ) + proj)


def gemma_activations(m: int, k: int, seed: int = 3, sub: int = 0) -> np.ndarray:
    return linear_activations(m, k, seed, sub=1000 + sub)[0]


# 70B-shaped linears: (K, N) in {(8192, 28672), (28672, 8192)}; W ~ N(0, 0.01);
# X ~ N(0, 1) with 0.1% of channels x50; M in {1, 16, 128, 4096}.
LLAMA70_SHAPES = ((8192, 28672), (28672, 8192))
LLAMA70_MS = (1, 16, 128, 4096)


def llama70_case(shape: int, m: int, seed: int = 5, with_x: bool = True) -> LinearCase:
    k, n = LLAMA70_SHAPES[shape]
    w = linear_weights(k, n, 0.01, seed, sub=shape)
    x, idx = (None, np.zeros(0, np.int64))
    if with_x:
        x, idx = linear_activations(m, k, seed, sub=10 * shape + m,
                                    outlier_count=round(0.001 * k), outlier_factor=50.0)
    return LinearCase(f"llama70_k{k}_n{n}_m{m}", x, w, idx)
