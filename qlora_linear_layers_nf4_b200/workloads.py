"""Seeded synthetic inputs for the NF4 / QLoRA-linear workloads.

This module only draws random numbers.  It holds none of the method's
arithmetic (no quantization, no matmul) and is the one piece of code that the
CPU oracle's tests and the CUDA path's tests share.

Recipe (every workload): NumPy Generator(PCG64(seed)), standard normal fp32
draws scaled by sigma, drawn in the order W, x, A, B, dy, bias.  BF16 tensors
are the round-to-nearest-even of those fp32 draws.
  W  ~ N(0, 0.02^2)   fp32, [N out, K in] row-major
  x  ~ N(0, 1)        bf16, [M, K]
  A  ~ N(0, 1/K)      bf16, [r, K]
  B  ~ N(0, 0.01^2)   bf16, [N, r]   (nonzero, so the adapter path is exercised)
  dy ~ N(0, 1)        bf16, [M, N]
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

W_SIGMA = 0.02
B_SIGMA = 0.01


@dataclass(frozen=True)
class LinearCase:
    """One QLoRA linear problem: y[M, N] = x[M, K] W'[N, K]^T + s t B^T."""
    name: str
    n: int              # out features
    k: int              # in features
    m: int              # tokens
    r: int
    alpha: float
    seed: int
    block_size: int = 64
    double_quant: bool = True
    with_bias: bool = False


# Tiny layer: W 256x256, 16 tokens, r=8, alpha=16, no double quant, seed 0.
TINY = LinearCase("tiny 256x256 M=16 r=8", n=256, k=256, m=16, r=8, alpha=16.0,
                  seed=0, double_quant=False)

# Quantize/dequantize of one 4096x4096 fp32 matrix, seed 1.
QUANT_SHAPE = (4096, 4096)
QUANT_SEED = 1

# Decode forward: W 4096x4096 with double quant, M in {1, 4, 16}, r=16, alpha=32.
DECODE = tuple(
    LinearCase(f"decode 4096x4096 M={m} r=16", n=4096, k=4096, m=m, r=16, alpha=32.0, seed=2)
    for m in (1, 4, 16)
)

# Prefill / training: gate_proj-like W 11008x4096, 4096 tokens, r=64, alpha=16.
PREFILL = LinearCase("prefill 11008x4096 M=4096 r=64", n=11008, k=4096, m=4096, r=64,
                     alpha=16.0, seed=3)

# One decoder block's seven targets, 2048 tokens, r=64, alpha=128.
BLOCK_TARGETS = (("q_proj", 4096, 4096), ("k_proj", 4096, 4096), ("v_proj", 4096, 4096),
                 ("o_proj", 4096, 4096), ("gate_proj", 11008, 4096),
                 ("up_proj", 11008, 4096), ("down_proj", 4096, 11008))
BLOCK = tuple(
    LinearCase(f"block {name} {n}x{k} M=2048 r=64", n=n, k=k, m=2048, r=64, alpha=128.0,
               seed=4 + i)
    for i, (name, n, k) in enumerate(BLOCK_TARGETS)
)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even, via torch."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class LinearInputs:
    case: LinearCase
    w: np.ndarray                 # fp32 [N, K]
    x: np.ndarray                 # bf16 bits [M, K]
    a: np.ndarray                 # bf16 bits [r, K]
    b: np.ndarray                 # bf16 bits [N, r]
    dy: np.ndarray                # bf16 bits [M, N]
    bias: np.ndarray | None = None  # bf16 bits [N]
    extra: dict = field(default_factory=dict)


def draw_linear(case: LinearCase, m: int | None = None) -> LinearInputs:
    """Draw W, x, A, B, dy (and bias) for one case, in that order."""
    m = case.m if m is None else m
    rng = np.random.Generator(np.random.PCG64(case.seed))
    w = (rng.standard_normal((case.n, case.k), dtype=np.float32) * np.float32(W_SIGMA))
    x = rng.standard_normal((m, case.k), dtype=np.float32)
    a = rng.standard_normal((case.r, case.k), dtype=np.float32) * np.float32(1.0 / np.sqrt(case.k))
    b = rng.standard_normal((case.n, case.r), dtype=np.float32) * np.float32(B_SIGMA)
    dy = rng.standard_normal((m, case.n), dtype=np.float32)
    bias = None
    if case.with_bias:
        bias = to_bf16_bits(rng.standard_normal(case.n, dtype=np.float32) * np.float32(0.1))
    out = LinearInputs(case, w.astype(np.float32), to_bf16_bits(x), to_bf16_bits(a),
                       to_bf16_bits(b), to_bf16_bits(dy), bias)
    # the fp32 draws themselves, for rounding to another compute dtype (f16)
    out.extra["f32"] = {"x": x, "a": a, "b": b, "dy": dy}
    return out


def draw_weight(shape, seed: int, sigma: float = W_SIGMA) -> np.ndarray:
    """An fp32 weight matrix ~ N(0, sigma^2) from its own seed."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(sigma)).astype(np.float32)
