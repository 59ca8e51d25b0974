"""GPU parity of awq_pseudo_quantize_pack and awq_dequant against the oracle:
bit-exact codes, packed words, scales, zeros and decoded weights."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import bits, dev, host, sample_rows
from workloads import make_packed_random, make_weight

pytestmark = pytest.mark.gpu


def degenerate_weight(rng) -> np.ndarray:
    """Rows whose groups hit the quantizer's special cases."""
    rows = [
        rng.normal(0, 0.02, (3, 512)),
        np.full((1, 512), 0.3), np.zeros((1, 512)), np.full((1, 512), -0.25),   # constant groups
        rng.uniform(0.1, 2.0, (2, 512)),                                         # all positive
        -rng.uniform(0.1, 2.0, (2, 512)),                                        # all negative
        rng.uniform(-1e-6, 1e-6, (2, 512)),                                      # fp16 subnormals
        rng.uniform(-6e4, 6e4, (2, 512)),                                        # near fp16 max
        np.round(rng.uniform(-8, 8, (3, 512))) / 2,                              # exact .5 ties
    ]
    return np.concatenate(rows).astype(np.float16)


def check_quantize(W: np.ndarray, zp: bool, rows=None):
    qg, sg, zg = awq.awq_pseudo_quantize_pack(dev(W), zero_point=zp)
    torch.cuda.synchronize()
    Wr = W if rows is None else W[rows]
    codes, scales, zeros = O.pseudo_quantize(Wr, 128, zp)
    # packed codes are [N, K/8]; scales and zero points are group-major [K/128, N]
    sel_rows = (lambda t: host(t)) if rows is None else (lambda t: host(t)[rows])
    sel_cols = (lambda t: host(t)) if rows is None else (lambda t: host(t)[:, rows])
    assert np.array_equal(bits(sel_rows(qg)), bits(O.pack(codes))), "packed codes differ"
    assert np.array_equal(bits(sel_cols(sg)), bits(scales)), "scales differ"
    if zp:
        assert np.array_equal(bits(sel_cols(zg)), bits(zeros)), "zero points differ"
    else:
        assert zg is None
    return qg, sg, zg


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(512, 512), (1, 128), (37, 256), (1000, 1024), (4096, 4096)])
def test_quantize_bit_exact(N, K, zp):
    W = make_weight(N, K, 0.02, 0.01, seed=N + K)
    check_quantize(W, zp)


@pytest.mark.parametrize("zp", [True, False])
def test_quantize_degenerate_groups(zp):
    W = degenerate_weight(np.random.default_rng(3))
    check_quantize(W, zp)


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K,sigma", [(14336, 4096, 0.02), (4096, 14336, 0.02), (28672, 8192, 0.015)])
def test_quantize_full_size_sampled_rows(N, K, sigma, zp):
    W = make_weight(N, K, sigma, 0.01, seed=0)
    check_quantize(W, zp, rows=sample_rows(N, 96))


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(512, 512), (3, 128), (1000, 1024), (4096, 14336)])
def test_dequant_bit_exact(N, K, zp):
    qweight, scales, zeros = make_packed_random(N, K, 128, zp, seed=N)
    Wd = awq.awq_dequant(dev(qweight), dev(scales), dev(zeros) if zp else None)
    ref = O.dequant(O.unpack(qweight), scales, zeros, 128)
    assert np.array_equal(bits(Wd), bits(ref))


@pytest.mark.parametrize("zp", [True, False])
def test_dequant_roundtrip_of_gpu_codes(zp):
    """Quantize then decode on the GPU equals the oracle's decode of its own codes."""
    W = make_weight(2048, 4096, 0.02, 0.01, seed=5)
    qg, sg, zg = awq.awq_pseudo_quantize_pack(dev(W), zero_point=zp)
    Wd = awq.awq_dequant(qg, sg, zg)
    codes, scales, zeros = O.pseudo_quantize(W, 128, zp)
    assert np.array_equal(bits(Wd), bits(O.dequant(codes, scales, zeros, 128)))


def test_quantize_empty_rows_is_a_no_op():
    W = torch.empty((0, 256), dtype=torch.float16, device="cuda")
    q, s, z = awq.awq_pseudo_quantize_pack(W)
    assert q.shape == (0, 32) and s.shape == (2, 0) and z.shape == (2, 0)


def test_quantize_rejects_bad_group():
    W = torch.zeros((8, 200), dtype=torch.float16, device="cuda")
    with pytest.raises(awq.AwqError, match="SHAPE"):
        awq.awq_pseudo_quantize_pack(W)
