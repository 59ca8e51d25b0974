"""GPU parity of the activation-aware scale search (awq_search_scale) and of
awq_apply_scale against the oracle's restatement of the same steps.

Tolerances: the per-channel statistics are fp32 sums taken in a different
order on each side, so a scale differs from the oracle's by at most a few
fp32 ulps (rtol 1e-5). A loss is a mean of squared differences of two fp16
outputs; the GPU's fp32-accumulated products may round an output to the
neighbouring fp16 value where the oracle's float64 sum does not, which moves
a loss by far less than 1e-3 relative (the test allows 2e-3). The chosen grid
point must be the oracle's, or tie with it within that tolerance."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import bits, dev, host
from workloads import make_weight

pytestmark = pytest.mark.gpu


def salient_inputs(Ms, K, seed, n_salient=8, factor=20.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((Ms, K), dtype=np.float32)
    X[:, rng.choice(K, n_salient, replace=False)] *= factor
    return X.astype(np.float16)


@pytest.mark.parametrize("N,K,Ms,zp,duo", [
    (128, 512, 32, True, True),      # product on the GEMM path (Ms > 16)
    (256, 1024, 8, True, True),      # product on the GEMV path
    (256, 1024, 64, False, True),    # symmetric
    (128, 512, 16, True, False),     # activation statistic only
])
def test_search_matches_the_oracle(N, K, Ms, zp, duo):
    W = make_weight(N, K, 0.02, 0.0, seed=11)
    X = salient_inputs(Ms, K, seed=12)
    n_grid = 10
    s_ref, losses_ref, best_ref = O.search_scale(W, X, 128, zp, n_grid, duo)
    s, losses = awq.awq_search_scale(dev(W), dev(X), zero_point=zp, n_grid=n_grid, duo=duo)
    losses = host(losses).astype(np.float64)
    np.testing.assert_allclose(losses, losses_ref, rtol=2e-3, atol=0)
    best = int(np.argmin(losses))
    assert best == best_ref or abs(losses_ref[best] - losses_ref[best_ref]) <= 2e-3 * losses_ref[best_ref]
    s_expect = O.candidate_scales(O.act_mean_abs(X), O.weight_norm_mean(W), best / n_grid, duo)
    np.testing.assert_allclose(host(s), s_expect, rtol=1e-5, atol=0)
    # repeated call: same bits
    s2, l2 = awq.awq_search_scale(dev(W), dev(X), zero_point=zp, n_grid=n_grid, duo=duo)
    assert np.array_equal(bits(host(s2)), bits(host(s))) and np.array_equal(bits(host(l2)), bits(losses.astype(np.float32)))


def test_search_helps_on_salient_channels():
    """The chosen scaling lowers the output error well below s = 1 (grid
    point 0 without duo scaling), as the oracle pin shows for the method."""
    W = make_weight(256, 1024, 0.02, 0.0, seed=21)
    X = salient_inputs(32, 1024, seed=22)
    _, losses = awq.awq_search_scale(dev(W), dev(X), n_grid=20, duo=True)
    _, plain = awq.awq_search_scale(dev(W), dev(X), n_grid=1, duo=False)
    losses = host(losses)
    assert int(np.argmin(losses)) > 0
    assert losses.min() < 0.8 * host(plain)[0]


def test_apply_scale_is_bit_exact():
    W = make_weight(96, 512, 0.02, 0.0, seed=31)
    s = np.random.default_rng(32).uniform(0.25, 4.0, 512).astype(np.float32)
    out = host(awq.awq_apply_scale(dev(W), dev(s)))
    want = (W.astype(np.float32) * s[None, :]).astype(np.float16)
    assert np.array_equal(bits(out), bits(want))
