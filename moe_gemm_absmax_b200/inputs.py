"""Seeded synthetic inputs for the W8A8 linear / MoE workloads.

This module holds random draws and their layout only; none of the method's
arithmetic (no quantization, no GEMM, no routing).  Both the CUDA path and
the CPU oracle take their inputs from here.  The casts of fp32 draws to
bf16 use torch's round-to-nearest-even conversion; that is part of making
the input, not of the method.

Recipe (numpy ``default_rng(seed)``; draws in fp32):
  * activations X ~ N(0, 1), then a set of outlier channels (columns drawn
    without replacement) multiplied by a factor, then cast to bf16;
  * weights W ~ N(0, 0.02) (0.02 is the standard deviation), fp32;
  * router logits ~ N(0, 1), cast to bf16.
"""
from __future__ import annotations

import numpy as np
import torch

# Workload shapes (dense Qwen3.6-27B-class linears, Qwen3.6-35B-A3B-class experts).
GATE_UP = dict(K=5120, N=34816)
DOWN = dict(K=17408, N=5120)
MOE = dict(E=256, H=2048, I=512, topk=8)
HADAMARD = dict(K=2048, N=4096)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round to nearest even."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(rng: np.random.Generator, M: int, K: int, n_outlier: int, factor: float) -> np.ndarray:
    x = rng.standard_normal((M, K), dtype=np.float32)
    if n_outlier > 0:
        cols = rng.choice(K, n_outlier, replace=False)
        x[:, cols] *= np.float32(factor)
    return x


def weights(rng: np.random.Generator, shape, std: float = 0.02) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


def outlier_count(K: int, frac: float = 0.001) -> int:
    """0.1 % of the channels: 5 of 5120, 17 of 17408."""
    return int(K * frac)


def tiny_linear(seed: int = 0, M: int = 16, K: int = 512, N: int = 512):
    """X bf16 [16,512] with 2 outlier columns x20, W fp32 [512,512]; row 0 is
    all zero and row 1 has a single nonzero element."""
    rng = np.random.default_rng(seed)
    x = activations(rng, M, K, 2, 20.0)
    x[0, :] = 0.0
    x[1, :] = 0.0
    x[1, 5] = -2.5
    w = weights(rng, (N, K))
    return to_bf16_bits(x), w


def dense_linear(seed: int, M: int, K: int, N: int, n_outlier: int | None = None,
                 factor: float = 30.0, with_weights: bool = True):
    """Decode- and prefill-shaped linears: 0.1 % outlier channels x30."""
    rng = np.random.default_rng(seed)
    if n_outlier is None:
        n_outlier = outlier_count(K)
    x = activations(rng, M, K, n_outlier, factor)
    w = weights(rng, (N, K)) if with_weights else None
    return to_bf16_bits(x), w


def moe_layer(seed: int, T: int, E: int = 256, H: int = 2048, I: int = 512,
              with_weights: bool = True):
    """Routed MoE layer: x ~ N(0,1) bf16 [T,H] (no outliers), router logits
    ~ N(0,1) bf16 [T,E], w13 fp32 [E,2I,H] (row 2i gate_i, row 2i+1 up_i),
    w2 fp32 [E,H,I]."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H), dtype=np.float32)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    w13 = weights(rng, (E, 2 * I, H)) if with_weights else None
    w2 = weights(rng, (E, H, I)) if with_weights else None
    return to_bf16_bits(x), to_bf16_bits(logits), w13, w2


def hadamard_linear(seed: int, M: int, K: int = 2048, N: int = 4096,
                    n_outlier: int = 20, factor: float = 50.0):
    """FWHT128-domain linear: X bf16 [M,K] with 20 heavy outlier channels x50;
    W ~ N(0,0.02) [N,K] cast to bf16 (a bf16 checkpoint)."""
    rng = np.random.default_rng(seed)
    x = activations(rng, M, K, n_outlier, factor)
    w = weights(rng, (N, K))
    return to_bf16_bits(x), to_bf16_bits(w)


def moe_weights(seed: int, E: int = 256, H: int = 2048, I: int = 512):
    """Expert weights drawn from their own stream, so that one set serves every
    token count: w13 fp32 [E,2I,H] (row 2i gate_i, row 2i+1 up_i), w2 fp32 [E,H,I]."""
    rng = np.random.default_rng([seed, 1])
    return weights(rng, (E, 2 * I, H)), weights(rng, (E, H, I))


def moe_tokens(seed: int, T: int, E: int = 256, H: int = 2048):
    """x ~ N(0,1) bf16 [T,H] and router logits ~ N(0,1) bf16 [T,E]."""
    rng = np.random.default_rng([seed, 2, T])
    x = rng.standard_normal((T, H), dtype=np.float32)
    logits = rng.standard_normal((T, E), dtype=np.float32)
    return to_bf16_bits(x), to_bf16_bits(logits)
