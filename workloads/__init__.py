"""Seeded synthetic inputs and the named workloads of the W4A16 linear layer.

This module only draws random numbers and names shapes. It holds none of the
quantization or matmul arithmetic, so both the CPU oracle side and the CUDA
side can take their inputs from it.

Input recipe (one ``numpy.random.default_rng(seed)`` stream per layer, draw
order fixed):

1. W: ``standard_normal((N, K), float32) * sigma``.
2. Salient input channels (when asked): ``ceil(frac * K)`` column indices
   drawn with ``rng.choice(K, n, replace=False)``; those columns of W are
   multiplied by 10. The AWQ pages describe a small fraction of
   activation-salient channels that dominate the error; the 1 % x10 recipe
   stands in for them since no trained weights are available.
3. W is cast to fp16 (round to nearest even).
4. x: ``standard_normal((M, K), float32)`` cast to fp16.

W depends only on (N, K, sigma, salient, seed), so a sweep over M reuses W.
Llama-3-8B / 70B layer shapes stand in for the pages' models (no checkpoint
is loaded; weights are random).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SALIENT_SCALE = 10.0


def make_weight(N: int, K: int, sigma: float, salient_frac: float = 0.0,
                seed: int = 0, rng: np.random.Generator | None = None) -> np.ndarray:
    """fp16 W[N, K] per steps 1-3 of the recipe."""
    rng = np.random.default_rng(seed) if rng is None else rng
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(sigma)
    if salient_frac > 0.0 and K > 0:
        n_sal = int(math.ceil(salient_frac * K))
        idx = rng.choice(K, size=n_sal, replace=False)
        W[:, idx] *= np.float32(SALIENT_SCALE)
    return W.astype(np.float16)


def make_activation(M: int, K: int, rng: np.random.Generator) -> np.ndarray:
    """fp16 x[M, K] ~ N(0, 1) (step 4)."""
    return rng.standard_normal((M, K), dtype=np.float32).astype(np.float16)


def make_layer(N: int, K: int, M: int, sigma: float, salient_frac: float = 0.0,
               seed: int = 0):
    """(W fp16 [N, K], x fp16 [M, K]) drawn in the recipe's order from one
    generator."""
    rng = np.random.default_rng(seed)
    W = make_weight(N, K, sigma, salient_frac, rng=rng)
    x = make_activation(M, K, rng)
    return W, x


def make_packed_random(N: int, K: int, group_size: int = 128, zero_point: bool = True,
                       seed: int = 0, scale_lo: float = 1e-3, scale_hi: float = 4e-3):
    """Random packed weights without any quantizer: uniform int32 words (every
    bit pattern is a valid set of eight 4-bit codes), fp16 scales uniform in
    [scale_lo, scale_hi], zero points uniform integers 0..15 stored as fp16;
    scales and zeros are group-major [K/group_size, N].
    Used where a test wants arbitrary codes rather than codes of some W."""
    rng = np.random.default_rng(seed)
    words = rng.integers(0, 2 ** 32, size=(N, K // 8), dtype=np.uint64).astype(np.uint32)
    qweight = words.view(np.int32)
    G = K // group_size
    scales = rng.uniform(scale_lo, scale_hi, size=(G, N)).astype(np.float16)
    zeros = rng.integers(0, 16, size=(G, N)).astype(np.float16) if zero_point else None
    return qweight, scales, zeros


@dataclass(frozen=True)
class LayerShape:
    name: str
    N: int
    K: int


@dataclass(frozen=True)
class Workload:
    """One named configuration: shapes, batch sizes, weight distribution."""
    name: str
    shapes: tuple
    Ms: tuple
    sigma: float
    salient_frac: float
    variants: tuple = ("asym",)
    notes: str = ""


LLAMA3_8B_DECODE = (
    LayerShape("q_proj", 4096, 4096),
    LayerShape("gate_proj", 14336, 4096),
    LayerShape("up_proj", 14336, 4096),
    LayerShape("down_proj", 4096, 14336),
)

WORKLOADS = {
    "single_512": Workload(
        "single_512", (LayerShape("linear", 512, 512),), (1,), 0.02, 0.0,
        notes="single W4A16 linear 512x512, M=1, asym g128, seed 0"),
    "llama3_8b_decode": Workload(
        "llama3_8b_decode", LLAMA3_8B_DECODE, (1,), 0.02, 0.01,
        notes="Llama-3-8B-shaped decode layers, M=1, 1% salient input channels x10"),
    "decode_sweep": Workload(
        "decode_sweep", (LayerShape("gate_proj", 14336, 4096), LayerShape("down_proj", 4096, 14336)),
        (1, 2, 4, 8, 16), 0.02, 0.0, variants=("asym", "sym"),
        notes="small-batch decode sweep, asym and sym"),
    "prefill": Workload(
        "prefill", (LayerShape("q_proj", 4096, 4096), LayerShape("gate_proj", 14336, 4096)),
        (128, 512, 2048), 0.02, 0.0,
        notes="prefill GEMM; M in {128, 512} locate the GEMV/GEMM crossover"),
    "llama3_70b": Workload(
        "llama3_70b", (LayerShape("qo_proj", 8192, 8192), LayerShape("gate_up_proj", 28672, 8192),
                       LayerShape("down_proj", 8192, 28672)),
        (1, 8, 2048), 0.015, 0.01,
        notes="Llama-3-70B-shaped layers, 1% salient input channels x10"),
}
