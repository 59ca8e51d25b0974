"""Pins of the oracle's fused gate/up projection (no GPU).

The oracle's SiLU, its gate*up product and the interleaved weight layout are
checked against things other than themselves: algebraic identities of SiLU,
an independent formula for the sigmoid, a per-element brute force with the
math module, and explicit indices of the layout.
"""
import math

import numpy as np
import pytest

from oracle import awq_oracle as O


def test_silu_identities():
    v = np.linspace(-30.0, 30.0, 601)
    s = O.silu_f64(v)
    assert O.silu_f64(np.array([0.0]))[0] == 0.0
    # silu(v) - silu(-v) = v (sigmoid(v) + sigmoid(-v) = 1)
    np.testing.assert_allclose(s - O.silu_f64(-v), v, rtol=0, atol=1e-12)
    # independent formulas for the sigmoid: (1 + tanh(v / 2)) / 2 for v >= 0,
    # e^v / (1 + e^v) for v < 0 (each free of cancellation on its side)
    pos, neg = v >= 0, v < 0
    np.testing.assert_allclose(s[pos], v[pos] * 0.5 * (1.0 + np.tanh(v[pos] / 2.0)), rtol=1e-13, atol=0)
    np.testing.assert_allclose(s[neg], v[neg] * np.exp(v[neg]) / (1.0 + np.exp(v[neg])), rtol=1e-13, atol=0)
    # tails: silu(v) -> v for large v, -> 0 from below for very negative v
    assert abs(O.silu_f64(np.array([60.0]))[0] - 60.0) < 1e-20 + 60.0 * 1e-15
    t = O.silu_f64(np.array([-60.0, -1000.0]))
    assert t[0] < 0 and abs(t[0]) < 1e-23 and t[1] == 0.0


def test_gate_up_silu_matches_brute_force():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 8)).astype(np.float16)
    Wg = (rng.standard_normal((5, 8)) * 0.5).astype(np.float16)
    Wu = (rng.standard_normal((5, 8)) * 0.5).astype(np.float16)
    h = O.gate_up_silu_f64(x, Wg, Wu)
    for m in range(3):
        for n in range(5):
            g = sum(float(x[m, k]) * float(Wg[n, k]) for k in range(8))
            u = sum(float(x[m, k]) * float(Wu[n, k]) for k in range(8))
            want = g / (1.0 + math.exp(-g)) * u
            assert abs(h[m, n] - want) <= 1e-12 * max(1.0, abs(want))


def test_interleave_layout_indices():
    g = np.arange(32 * 3).reshape(32, 3)
    u = 1000 + np.arange(32 * 3).reshape(32, 3)
    out = O.interleave_gate_up(g, u)
    assert out.shape == (64, 3)
    # tile order: gate 0..15, up 0..15, gate 16..31, up 16..31
    assert np.array_equal(out[0:16], g[0:16]) and np.array_equal(out[16:32], u[0:16])
    assert np.array_equal(out[32:48], g[16:32]) and np.array_equal(out[48:64], u[16:32])
    # along axis 1 (group-major scales [G, N])
    sg, su = g.T.copy(), u.T.copy()
    assert np.array_equal(O.interleave_gate_up(sg, su, axis=1), out.T)
    with pytest.raises(ValueError):
        O.interleave_gate_up(g[:24], u[:24])


def test_interleaved_linear_then_pairs_is_gate_up():
    """The fused layer read as one linear over 2N rows, then silu(tile 2j) *
    tile 2j+1 row by row, equals silu(gate) * up: the layout and the product
    compose as the fused kernels assume."""
    rng = np.random.default_rng(6)
    N, K = 32, 256
    Wg = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    Wu = (rng.standard_normal((N, K)) * 0.02).astype(np.float16)
    x = rng.standard_normal((2, K)).astype(np.float16)
    Y = O.matmul_f64(x, O.interleave_gate_up(Wg, Wu))
    h = np.empty((2, N))
    for j in range(N // 16):
        h[:, 16 * j:16 * j + 16] = O.silu_f64(Y[:, 32 * j:32 * j + 16]) * Y[:, 32 * j + 16:32 * j + 32]
    np.testing.assert_allclose(h, O.gate_up_silu_f64(x, Wg, Wu), rtol=1e-13, atol=1e-15)
