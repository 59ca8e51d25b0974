"""GPU parity of awq_gemm (tcgen05 tensor-core path) against the float64 oracle.

Small and ragged shapes are compared on every output; the prefill and 70B
configurations at full size on sampled output channels (all rows of x)."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import (activations, assert_close, bits, dev, host, oracle_layer, sample_rows)
from workloads import make_packed_random, make_weight

pytestmark = pytest.mark.gpu


def run_gemm(x, qweight, scales, zeros):
    y = awq.awq_gemm(dev(x), dev(qweight), dev(scales), dev(zeros) if zeros is not None else None)
    torch.cuda.synchronize()
    return host(y)


@pytest.fixture(autouse=True)
def no_device_error():
    yield
    assert awq.awq_device_error() == 0, "a pipeline wait inside awq_gemm timed out"


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K,Ms", [
    (512, 512, (1, 16, 17, 128, 129, 300)),
    (256, 128, (128,)),                 # one tile, one k-block pair
    (40, 256, (7, 200)),                # ragged N smaller than a tile
    (1000, 1024, (128, 257)),           # ragged N and M
    (4096, 4096, (128,)),
])
def test_gemm_full_compare(N, K, Ms, zp):
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, zp)
    for M in Ms:
        x = activations(M, K, seed=M)
        y = run_gemm(x, qweight, scales, zeros)
        assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M} zp={zp}")


def test_gemm_odd_n_scalar_epilogue():
    """N not a multiple of 8 takes the element-wise store path."""
    qweight, scales, zeros = make_packed_random(301, 512, 128, True, seed=9)
    Wd = O.dequant(O.unpack(qweight), scales, zeros, 128)
    x = activations(130, 512, seed=2)
    assert_close(run_gemm(x, qweight, scales, zeros), O.matmul_f64(x, Wd), "N=301")


@pytest.mark.parametrize("N,K,M", [(4000, 256, 1300), (2999, 256, 1300), (3000, 384, 2000)])
def test_gemm_cta_pairs_many_tiles(N, K, M):
    """Whole tiles on CTA pairs: 72 to 96 tiles of 256 x 256 (some pairs take
    two, through both accumulators), ragged last row and channel tiles (the
    second CTA of the last row tile has no rows of x), N not a multiple of 8.
    Full compare, and bit-identical on a second call."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(M, K, seed=60 + M)
    y = run_gemm(x, qweight, scales, zeros)
    assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M}")
    assert np.array_equal(bits(y), bits(run_gemm(x, qweight, scales, zeros)))


def test_gemm_last_partial_wave_goes_to_k_slices():
    """150 tiles on 148 SMs: 148 on the persistent grid, the last 2 (the
    ragged last channel tile, both row tiles, the second only partly filled)
    in a second launch with K split over clusters. Full compare."""
    N, K, M = 19192, 1024, 500
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(M, K, seed=71)
    y = run_gemm(x, qweight, scales, zeros)
    assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M}")


@pytest.mark.parametrize("N,K,M", [(512, 4096, 200), (1024, 2048, 64), (2048, 8192, 129), (4096, 4096, 17)])
def test_gemm_k_slices_over_a_cluster(N, K, M):
    """Few tiles: K is split over a cluster of 4 or 8 CTAs per tile and the slices
    are summed through distributed shared memory (M = 200 and 129: the upper
    half of the tile is partly filled). Full compare, and bit-identical on a
    second call."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(M, K, seed=50 + M)
    y = run_gemm(x, qweight, scales, zeros)
    assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M}")
    assert np.array_equal(bits(y), bits(run_gemm(x, qweight, scales, zeros)))


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_gemm_prefill_sampled(N, K):
    """Prefill: M in {128, 512, 2048}; sampled output channels, every row of x."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.0, True)
    cols = sample_rows(N, 384)
    for M in (128, 512, 2048):
        x = activations(M, K, seed=30 + M)
        y = run_gemm(x, qweight, scales, zeros)
        assert_close(y[:, cols], O.matmul_f64(x, Wd[cols]), f"N={N} K={K} M={M}")


@pytest.mark.parametrize("N,K", [(8192, 8192), (28672, 8192), (8192, 28672)])
def test_gemm_llama3_70b_sampled(N, K):
    W = make_weight(N, K, 0.015, 0.01, seed=0)
    qg, sg, zg = awq.awq_pseudo_quantize_pack(dev(W), zero_point=True)
    cols = sample_rows(N, 256)
    codes, scales, zeros = O.pseudo_quantize(W[cols], 128, True)
    assert np.array_equal(bits(host(qg)[cols]), bits(O.pack(codes)))
    Wd = O.dequant(codes, scales, zeros, 128)
    x = activations(2048, K, seed=40)
    y = host(awq.awq_gemm(dev(x), qg, sg, zg))
    assert_close(y[:, cols], O.matmul_f64(x, Wd), f"N={N} K={K} M=2048")


def test_gemm_matches_gemv_at_small_m():
    _, qweight, scales, zeros, Wd = oracle_layer(4096, 4096, 0.02, 0.01, True)
    for M in (1, 8, 16):
        x = activations(M, 4096, seed=M)
        ws = awq.alloc_workspace(M, 4096, 4096, True)
        yv = host(awq.awq_gemv(dev(x), dev(qweight), dev(scales), dev(zeros), workspace=ws))
        yg = run_gemm(x, qweight, scales, zeros)
        ref = O.matmul_f64(x, Wd)
        assert_close(yv, ref, f"gemv M={M}")
        assert_close(yg, ref, f"gemm M={M}")


def test_gemm_is_deterministic():
    _, qweight, scales, zeros, _ = oracle_layer(1000, 1024, 0.02, 0.01, True)
    x = activations(300, 1024, seed=1)
    a = bits(run_gemm(x, qweight, scales, zeros))
    b = bits(run_gemm(x, qweight, scales, zeros))
    assert np.array_equal(a, b)


def test_gemm_empty_batch():
    _, qweight, scales, zeros, _ = oracle_layer(512, 512, 0.02, 0.01, True)
    y = awq.awq_gemm(torch.empty((0, 512), dtype=torch.float16, device="cuda"), dev(qweight), dev(scales),
                     dev(zeros))
    assert y.shape == (0, 512)


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 4096), (6144, 4096), (4096, 14336)])
def test_gemm_small_batches_around_the_crossover(N, K, zp):
    """Prefill batches between the GEMV range and a full 256-row tile of x
    (M = 17 .. 128, and 160 / 256 on both sides of one x tile), where the
    product may take 128-channel tiles: every output of sampled channels
    against the float64 oracle, both zero-point variants, and the same bits
    on a second call."""
    W = make_weight(N, K, 0.02, 0.01, seed=21)
    codes, scales, zeros = O.pseudo_quantize(W, 128, zp)
    qweight = O.pack(codes)
    rows = sample_rows(N, 256, seed=N)
    Wd = O.dequant(codes[rows], scales[:, rows], zeros[:, rows] if zp else None, 128)
    q, s, z = dev(qweight), dev(scales), dev(zeros) if zp else None
    for M in (17, 24, 32, 48, 64, 96, 128, 160, 256):
        xh = activations(M, K, seed=M)
        x = dev(xh)
        y = awq.awq_gemm(x, q, s, z)
        y2 = awq.awq_gemm(x, q, s, z)
        torch.cuda.synchronize()
        assert_close(host(y)[:, rows], O.matmul_f64(xh, Wd), f"N={N} K={K} M={M} zp={zp}")
        assert np.array_equal(bits(y), bits(y2)), f"M={M}: second call differs"


@pytest.mark.parametrize("M", [24, 96, 128])
def test_gemm_small_batches_fused_gate_up(M):
    """The fused SiLU epilogue on 128-channel tiles (8 gate/up tile pairs per
    256 channels, 4 per 128): against the float64 oracle of silu(gate) * up."""
    N, K = 5632, 2048
    Wg = make_weight(N, K, 0.02, 0.0, seed=31)
    Wu = make_weight(N, K, 0.02, 0.0, seed=32)
    cg, sg, zg = O.pseudo_quantize(Wg, 128, True)
    cu, su, zu = O.pseudo_quantize(Wu, 128, True)
    q, s, z = awq.awq_interleave_gate_up(dev(O.pack(cg)), dev(sg), dev(zg), dev(O.pack(cu)), dev(su), dev(zu))
    xh = activations(M, K, seed=5)
    y = host(awq.awq_gemm(dev(xh), q, s, z, silu_mul=True))
    ref = O.gate_up_silu_f64(xh, O.dequant(cg, sg, zg, 128), O.dequant(cu, su, zu, 128))
    assert_close(y, ref, f"fused M={M}")
