"""Pins of the oracle's clip search (no GPU): the clipping by hand, ratio 1
as the identity, the Gram form of the output error against the direct
product, and that the search helps on groups with an outlier."""

import os

import numpy as np

from oracle import awq_oracle as O
from workloads import make_weight


def test_clip_groups_by_hand():
    W = np.zeros((1, 128), dtype=np.float16)
    W[0, :4] = [4.0, -2.0, 1.0, -4.0]
    C = O.clip_groups(W, np.array([[0.5]], np.float32))
    assert list(C[0, :4]) == [2.0, -2.0, 1.0, -2.0]
    assert np.array_equal(O.clip_groups(W, np.ones((1, 1), np.float32)), W)   # ratio 1: unchanged


def test_gram_error_equals_direct_output_error():
    rng = np.random.default_rng(3)
    W = make_weight(8, 256, 0.02, 0.0, seed=4)
    X = rng.standard_normal((16, 256)).astype(np.float16)
    ratios, errs = O.search_clip(W, X, n_grid=3)
    codes, sc, z = O.pseudo_quantize(W)                   # grid point 0 is ratio 1: no clip
    D = W.astype(np.float64) - O.dequant(codes, sc, z).astype(np.float64)
    Xf = X.astype(np.float64)
    for j in range(2):
        sl = slice(128 * j, 128 * j + 128)
        direct = ((Xf[:, sl] @ D[:, sl].T) ** 2).sum(axis=0)    # [N]
        np.testing.assert_allclose(errs[0, j], direct, rtol=1e-10)


def test_search_clips_outlier_groups():
    """A group with one extreme weight: clipping it trades a large error on
    one weight for finer steps on the rest, and the search takes it."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    W[:, 7] = 0.5 * np.sign(rng.standard_normal(64))    # one outlier per row in group 0
    W = W.astype(np.float16)
    X = rng.standard_normal((64, 256)).astype(np.float16)
    X[:, 7] *= 0.01                                        # ... on an input channel that barely matters
    ratios, errs = O.search_clip(W, X, n_grid=10)
    assert np.all(ratios <= 1.0) and np.all(ratios > 0.5)
    assert np.mean(ratios[0] < 1.0) > 0.9                  # group 0 is clipped for almost every row
    best = errs.min(axis=0)
    assert np.all(best <= errs[0]) and best[0].sum() < 0.5 * errs[0, 0].sum()


def test_clip_grid_hand_worked(golden_dir):
    """The ratio grid of search_clip against the case worked by hand in
    search_readings_worked.txt: with n_grid = 4 and max_shrink = 1/2 the grid
    is 1, 7/8, 3/4, 5/8, and ratio 3/4 puts every weight that matters exactly
    on the quantization grid (error 0), so every row picks it."""
    row = None
    with open(os.path.join(golden_dir, "search_readings_worked.txt")) as f:
        for line in f:
            parts = line.split()
            if parts and parts[0] == "clip":
                row = parts[1:]
    n_grid, shrink, outlier, best_i, best_r = int(row[0]), float(row[1]), float(row[2]), int(row[3]), float(row[4])
    rng = np.random.default_rng(8)
    N = 16
    W = (rng.integers(-7, 8, (N, 128)) / 16.0).astype(np.float16)
    W[:, 0], W[:, 1] = outlier, -outlier
    X = rng.standard_normal((256, 128)).astype(np.float16)
    X[:, :2] = 0.0
    ratios, errs = O.search_clip(W, X, n_grid=n_grid, max_shrink=shrink)
    assert errs.shape == (n_grid, 1, N)
    assert np.all(errs[best_i] == 0.0)
    assert np.all(np.delete(errs, best_i, axis=0) > 0.0)
    assert np.all(ratios == np.float32(best_r))
