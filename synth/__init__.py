"""Seeded synthetic inputs for the BitLinear workloads.

This module only draws inputs.  It holds none of the layer's arithmetic (no
scales, codes, rounding rules or products), and it serves both the CUDA path
and the CPU oracle, which otherwise share nothing.

Workloads (shapes and distributions follow the decode/prefill settings the
BitNet b1.58 pages describe for 2B-, 7B- and 100B-class models; the weights
are random N(0, 0.02) because no trained checkpoints are used):

  single    M=8,  K=512 -> N=512, W ~ N(0, 0.02) fp32, x ~ N(0, 1) fp32
  block2b   M=1, the seven linears of a 2B-class block (gate/up, down, q/o,
            k/v), x ~ N(0, 1) with 1% of elements scaled x20, cast to bf16
  7b        M in {1, 4, 16} x {4096->11008, 11008->4096, 4096->4096}, bf16 x
  prefill   M=2048 x {2560->6912, 6912->2560}, bf16 x, bf16 out
  sweep100b M=1, 80 layers x {8192->28672 x2, 28672->8192, 8192->8192 x2,
            8192->1024 x2}; weights generated on each side by the
            counter-based recipe in ``synth.device`` / the oracle
"""
from __future__ import annotations

import numpy as np

SIGMA_W = 0.02

# (K, N, name) for each linear of one 2B-class block, in forward order.
BLOCK2B = [
    (2560, 6912, "gate"),
    (2560, 6912, "up"),
    (6912, 2560, "down"),
    (2560, 2560, "q"),
    (2560, 2560, "o"),
    (2560, 640, "k"),
    (2560, 640, "v"),
]

SHAPES_7B = [(4096, 11008, "up"), (11008, 4096, "down"), (4096, 4096, "qkvo")]
M_7B = (1, 4, 16)

PREFILL = [(2560, 6912, "gate_up"), (6912, 2560, "down")]
M_PREFILL = 2048

# One 100B-class layer: (K, N, name); the sweep runs 80 such layers.
LAYER100B = [
    (8192, 28672, "gate"),
    (8192, 28672, "up"),
    (28672, 8192, "down"),
    (8192, 8192, "q"),
    (8192, 8192, "o"),
    (8192, 1024, "k"),
    (8192, 1024, "v"),
]
LAYERS100B = 80


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def weights(N: int, K: int, seed: int, sigma: float = SIGMA_W) -> np.ndarray:
    """fp32 [N, K] weights ~ N(0, sigma^2), row-major like nn.Linear.weight."""
    w = rng(seed).standard_normal((N, K), dtype=np.float32)
    w *= np.float32(sigma)
    return w


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Cast fp32 values to bf16 (round to nearest even); returns uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(M: int, K: int, seed: int, dtype: str = "bf16", outlier_frac: float = 0.0,
                outlier_scale: float = 20.0) -> np.ndarray:
    """x ~ N(0, 1) [M, K]; a Bernoulli(outlier_frac) subset is multiplied by
    outlier_scale before the cast.  dtype 'f32' returns float32, 'bf16'
    returns the uint16 bit patterns of the bf16 values."""
    g = rng(seed)
    x = g.standard_normal((M, K), dtype=np.float32)
    if outlier_frac > 0.0:
        mask = g.random((M, K)) < outlier_frac
        x[mask] *= np.float32(outlier_scale)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(f"unknown dtype {dtype!r}")


def block2b_inputs(seed_base: int = 0, M: int = 1):
    """Weights and activations of the seven 2B-block linears (seed i per linear)."""
    out = []
    for i, (K, N, name) in enumerate(BLOCK2B):
        out.append(dict(name=name, K=K, N=N, W=weights(N, K, seed_base + i),
                        x=activations(M, K, 1000 + seed_base + i, "bf16", outlier_frac=0.01)))
    return out
