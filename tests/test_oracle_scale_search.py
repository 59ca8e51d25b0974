"""Pins of the oracle's activation-aware scale search (no GPU): the
statistics against hand-worked values, the candidate normalisation, the
alpha = 0 point against plain quantization, the scale invariance it relies
on, and that the search helps on inputs with salient channels."""

import numpy as np

from oracle import awq_oracle as O
from workloads import make_weight


def test_statistics_by_hand():
    X = np.array([[1.0, -2.0], [3.0, 0.5]], dtype=np.float16)
    np.testing.assert_array_equal(O.act_mean_abs(X), np.array([2.0, 1.25], dtype=np.float32))
    W = np.zeros((2, 128), dtype=np.float16)
    W[0, :2] = [2.0, -1.0]          # row 0: max 2 -> 1, 0.5
    W[1, :2] = [0.5, 0.25]          # row 1: max 0.5 -> 1, 0.5
    wm = O.weight_norm_mean(W)
    assert wm[0] == 1.0 and wm[1] == 0.5 and np.all(wm[2:] == 0.0)
    assert np.all(O.weight_norm_mean(np.zeros((3, 128), np.float16)) == 0.0)   # all-zero groups


def test_candidates_are_normalised():
    rng = np.random.default_rng(1)
    xm = rng.uniform(0.1, 5.0, 256).astype(np.float32)
    wm = rng.uniform(0.05, 1.0, 256).astype(np.float32)
    for a in (0.0, 0.3, 0.95):
        for duo in (True, False):
            s = O.candidate_scales(xm, wm, a, duo)
            assert s.dtype == np.float32 and np.all(s > 0)
            assert abs(float(s.max()) * float(s.min()) - 1.0) < 1e-5
    # alpha = 0 without duo scaling: every channel scale is 1
    assert np.all(O.candidate_scales(xm, wm, 0.0, False) == 1.0)


def test_alpha_zero_is_plain_quantization():
    W = make_weight(64, 256, 0.02, 0.0, seed=3)
    X = np.random.default_rng(4).standard_normal((8, 256), dtype=np.float32).astype(np.float16)
    s = O.candidate_scales(O.act_mean_abs(X), O.weight_norm_mean(W), 0.0, duo=False)
    y = O.scaled_output(W, X, s)
    codes, sc, z = O.pseudo_quantize(W)
    assert np.array_equal(y, O.matmul_f64(X, O.dequant(codes, sc, z)).astype(np.float16))


def test_scale_invariance_without_quantization():
    """(x / s) . (W diag(s))^T == x . W^T exactly for power-of-two s: the
    identity the search relies on (scaling moves error, not the function)."""
    rng = np.random.default_rng(5)
    W = rng.standard_normal((16, 64)).astype(np.float16)
    X = rng.standard_normal((4, 64)).astype(np.float16)
    s = np.float32(2.0) ** rng.integers(-3, 4, 64).astype(np.float32)
    Ws = (W.astype(np.float32) * s).astype(np.float16)
    Xs = (X.astype(np.float32) / s).astype(np.float16)
    assert np.array_equal(O.matmul_f64(Xs, Ws), O.matmul_f64(X, W))


def test_search_beats_plain_quantization_on_salient_channels():
    """Inputs whose few salient channels are 10x larger: the search finds an
    alpha > 0 whose output error is clearly below that of s = 1."""
    rng = np.random.default_rng(6)
    K = 512
    W = make_weight(128, K, 0.02, 0.0, seed=7)
    X = rng.standard_normal((32, K), dtype=np.float32)
    X[:, rng.choice(K, 8, replace=False)] *= 20.0
    X = X.astype(np.float16)
    s, losses, best = O.search_scale(W, X, n_grid=10, duo=True)
    plain = O.search_scale(W, X, n_grid=1, duo=False)[1][0]     # alpha = 0, no duo: s = 1
    assert best > 0 and losses[best] == losses.min()
    assert losses[best] < 0.8 * plain
