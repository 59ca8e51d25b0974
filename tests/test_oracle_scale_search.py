"""Pins of the oracle's activation-aware scale search (no GPU): the
statistics against hand-worked values, the candidate normalisation, the
alpha = 0 point against plain quantization, the scale invariance it relies
on, and that the search helps on inputs with salient channels."""

import os

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


def _golden_rows(golden_dir, kind):
    rows = []
    with open(os.path.join(golden_dir, "search_readings_worked.txt")) as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == kind:
                rows.append(parts[1:])
    return rows


def test_candidates_hand_worked(golden_dir):
    """candidate_scales against the values worked by hand in
    search_readings_worked.txt: four channels whose activation and weight
    statistics are powers of two, at alpha = 1/4 and 1/2, with and without
    duo scaling. The alpha = 1/4 rows tell the activation exponent alpha from
    1 - alpha and the weight exponent 1 - alpha from alpha; the duo rows tell
    dividing by the weight statistic from multiplying by it."""
    xm = np.array([16.0, 4.0, 1.0, 0.0625], dtype=np.float32)
    wm = np.array([0.0625, 1.0, 0.25, 1.0], dtype=np.float32)
    rows = _golden_rows(golden_dir, "candidates")
    assert len(rows) == 4
    for alpha, duo, *vals in rows:
        s = O.candidate_scales(xm, wm, float(alpha), bool(int(duo)))
        np.testing.assert_allclose(s, np.array(vals, dtype=np.float64), rtol=2e-6,
                                   err_msg=f"alpha={alpha} duo={duo}")


def test_candidate_ratios_do_not_depend_on_the_normalisation():
    """Between two channels with the same weight statistic the scales differ
    by exactly (x_i / x_j)^alpha, whatever the normaliser: 16 against 1 at
    alpha = 1/4 gives 2."""
    xm = np.array([16.0, 1.0, 3.0], dtype=np.float32)
    wm = np.array([0.5, 0.5, 0.2], dtype=np.float32)
    for duo in (False, True):
        s = O.candidate_scales(xm, wm, 0.25, duo)
        assert abs(float(s[0]) / float(s[1]) - 2.0) < 1e-6


def test_loss_hand_worked(golden_dir):
    """search_scale's loss at one grid point against the mean square worked by
    hand (5/8192); a mean absolute difference would give 3/128."""
    (w0, w1, w2, x0, x1, num, den), = _golden_rows(golden_dir, "loss")
    W = np.zeros((1, 128), dtype=np.float16)
    W[0, :3] = [float(w0), float(w1), float(w2)]
    X = np.zeros((2, 128), dtype=np.float16)
    X[0, 2], X[1, 2] = float(x0), float(x1)
    _, losses, best = O.search_scale(W, X, n_grid=1, duo=False)
    assert best == 0 and losses.shape == (1,)
    assert losses[0] == int(num) / int(den)
