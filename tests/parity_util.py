"""Shared helpers for the GPU parity tests: seeded layers quantized by the
oracle (cached per shape), host/device transfer, and the tolerance check.

Tolerance (floating-point outputs of the matmul): relative Frobenius error
<= 5e-3 and max abs error <= 1e-2 * max|y_ref| against the float64 oracle.
Codes, packed words, scales, zeros and decoded weights are compared bit for
bit."""

from __future__ import annotations

import functools

import numpy as np
import torch

from oracle import awq_oracle as O
from workloads import make_weight

REL_FROB_TOL = 5e-3
MAX_ABS_TOL = 1e-2


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bits(a) -> np.ndarray:
    a = host(a) if isinstance(a, torch.Tensor) else np.asarray(a)
    return a.view(np.uint16) if a.dtype == np.float16 else a.view(np.uint32)


def assert_close(y: np.ndarray, y_ref: np.ndarray, tag: str = ""):
    y64 = np.asarray(y, dtype=np.float64)
    assert np.all(np.isfinite(y64)), f"{tag}: non-finite output"
    rf = O.rel_frobenius(y64, y_ref)
    ma = O.max_abs_ratio(y64, y_ref)
    assert rf <= REL_FROB_TOL and ma <= MAX_ABS_TOL, f"{tag}: rel_frob={rf:.3e} max_abs={ma:.3e}"
    return rf, ma


@functools.lru_cache(maxsize=8)
def oracle_layer(N: int, K: int, sigma: float, salient: float, zp: bool, seed: int = 0):
    """(W, qweight, scales, zeros, W') from the seeded generator and the oracle."""
    W = make_weight(N, K, sigma, salient, seed=seed)
    codes, scales, zeros = O.pseudo_quantize(W, 128, zp)
    Wd = O.dequant(codes, scales, zeros, 128)
    return W, O.pack(codes), scales, zeros, Wd


def activations(M: int, K: int, seed: int = 100) -> np.ndarray:
    return np.random.default_rng(seed).standard_normal((M, K), dtype=np.float32).astype(np.float16)


def sample_rows(N: int, n: int, seed: int = 7) -> np.ndarray:
    """Sorted sample of n row indices, always including the first and last rows."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist()) | {0, N - 1}
    return np.array(sorted(rows), dtype=np.int64)
