"""GPU parity of the fused gate/up projection (AWQ_FLAG_SILU_MUL) against the
float64 oracle: h = silu(x . Wg'^T) * (x . Wu'^T), with the weights in the
interleaved 16-row tile layout built by awq_interleave_gate_up.

The layout itself is compared bit for bit with the oracle's; the products
with the matmul tolerance, on every output for small shapes and on sampled
output channels (every row of x) for the Llama-3-8B MLP shape."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import activations, assert_close, bits, dev, host, oracle_layer, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def no_device_error():
    yield
    assert awq.awq_device_error() == 0, "a pipeline wait timed out"


def fused_layer(N, K, zp, sigma=0.02):
    """Gate (seed 0) and up (seed 1) projections of N rows, quantized by the
    oracle, interleaved on the GPU; returns the device tensors and both W'."""
    _, qg, sg, zg, Wg = oracle_layer(N, K, sigma, 0.0, zp, 0)
    _, qu, su, zu, Wu = oracle_layer(N, K, sigma, 0.0, zp, 1)
    q, s, z = awq.awq_interleave_gate_up(dev(qg), dev(sg), dev(zg) if zp else None,
                                         dev(qu), dev(su), dev(zu) if zp else None)
    torch.cuda.synchronize()
    return q, s, z, Wg, Wu


@pytest.mark.parametrize("zp", [True, False])
def test_interleave_is_the_documented_layout(zp):
    N, K = 96, 512
    _, qg, sg, zg, _ = oracle_layer(N, K, 0.02, 0.0, zp, 0)
    _, qu, su, zu, _ = oracle_layer(N, K, 0.02, 0.0, zp, 1)
    q, s, z = awq.awq_interleave_gate_up(dev(qg), dev(sg), dev(zg) if zp else None,
                                         dev(qu), dev(su), dev(zu) if zp else None)
    assert np.array_equal(bits(q), bits(O.interleave_gate_up(qg, qu, axis=0)))
    assert np.array_equal(bits(s), bits(O.interleave_gate_up(sg, su, axis=1)))
    if zp:
        assert np.array_equal(bits(z), bits(O.interleave_gate_up(zg, zu, axis=1)))
    else:
        assert z is None


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(512, 512), (1024, 2048), (2048, 1024)])
def test_gemv_silu_mul_small_shapes(N, K, zp):
    """Few tiles: K is cut into slices whose partials meet in the workspace,
    and the last CTA of a gate/up tile pair applies silu * up."""
    q, s, z, Wg, Wu = fused_layer(N, K, zp)
    for M in (1, 3, 8, 16):
        x = activations(M, K, seed=M)
        ws = awq.alloc_workspace(M, 2 * N, K, zp, silu_mul=True)
        y = host(awq.awq_gemv(dev(x), q, s, z, workspace=ws, silu_mul=True))
        assert y.shape == (M, N)
        assert_close(y, O.gate_up_silu_f64(x, Wg, Wu), f"N={N} K={K} M={M} zp={zp}")


def test_gemv_silu_mul_llama3_8b_mlp():
    """Gate and up of Llama-3-8B (14336 x 4096 each): 1792 tiles, whole tiles
    per CTA, silu * up in the chunk epilogue. Sampled output channels."""
    N, K = 14336, 4096
    q, s, z, Wg, Wu = fused_layer(N, K, True)
    cols = sample_rows(N, 384)
    for M in (1, 4, 16):
        x = activations(M, K, seed=20 + M)
        y = host(awq.awq_gemv(dev(x), q, s, z, weights_static=True, silu_mul=True))
        assert_close(y[:, cols], O.gate_up_silu_f64(x, Wg[cols], Wu[cols]), f"M={M}")
        y2 = host(awq.awq_gemv(dev(x), q, s, z, silu_mul=True))
        assert np.array_equal(bits(y), bits(y2)), "weights_static changed the bits"


def test_gemv_noalloc_silu_mul_same_bits():
    N, K = 1024, 2048
    q, s, z, _, _ = fused_layer(N, K, True)
    x = dev(activations(2, K, seed=9))
    ws = awq.alloc_workspace(2, 2 * N, K, True, silu_mul=True)
    a = bits(awq.awq_gemv(x, q, s, z, workspace=ws, silu_mul=True))
    b = bits(awq.awq_gemv_noalloc(x, q, s, z, silu_mul=True))
    assert np.array_equal(a, b)


@pytest.mark.parametrize("zp", [True, False])
def test_gemm_silu_mul_small_shapes(zp):
    N, K = 1024, 1024
    q, s, z, Wg, Wu = fused_layer(N, K, zp)
    for M in (17, 128, 300):
        x = activations(M, K, seed=30 + M)
        y = host(awq.awq_gemm(dev(x), q, s, z, silu_mul=True))
        assert y.shape == (M, N)
        assert_close(y, O.gate_up_silu_f64(x, Wg, Wu), f"M={M} zp={zp}")


def test_gemm_silu_mul_llama3_8b_prefill():
    """M = 2048 on the fused 28672 x 4096 weights: 896 tiles of 256 x 256 on
    the persistent grid (each tile 8 gate/up tile pairs). Sampled channels,
    and bit-identical on a second call."""
    N, K = 14336, 4096
    q, s, z, Wg, Wu = fused_layer(N, K, True)
    cols = sample_rows(N, 256)
    x = activations(2048, K, seed=41)
    y = host(awq.awq_gemm(dev(x), q, s, z, silu_mul=True))
    assert_close(y[:, cols], O.gate_up_silu_f64(x, Wg[cols], Wu[cols]), "M=2048")
    y2 = host(awq.awq_gemm(dev(x), q, s, z, silu_mul=True))
    assert np.array_equal(bits(y), bits(y2))


def test_silu_mul_matches_separate_products_then_silu():
    """The fused call equals the unfused layer over the interleaved weights
    followed by silu(gate rows) * (up rows) in fp32: the same fp32 sums, one
    fp16 rounding at the end (GEMV, whole tiles)."""
    N, K = 14336, 4096
    q, s, z, _, _ = fused_layer(N, K, True)
    xh = activations(1, K, seed=77)
    h = host(awq.awq_gemv(dev(xh), q, s, z, silu_mul=True)).astype(np.float64)
    ref = O.gate_up_silu_f64(xh, *[oracle_layer(N, K, 0.02, 0.0, True, sd)[4] for sd in (0, 1)])
    assert_close(h, ref, "fused vs oracle")


@pytest.mark.parametrize("zp", [True, False])
def test_concat_rows_is_the_concatenation(zp):
    shapes = [(256, 512), (64, 512), (96, 512)]
    parts = [oracle_layer(n, k, 0.02, 0.0, zp, i) for i, (n, k) in enumerate(shapes)]
    q, s, z = awq.awq_concat_rows([(dev(p[1]), dev(p[2]), dev(p[3]) if zp else None) for p in parts])
    assert np.array_equal(bits(q), bits(np.concatenate([p[1] for p in parts], axis=0)))
    assert np.array_equal(bits(s), bits(np.concatenate([p[2] for p in parts], axis=1)))
    if zp:
        assert np.array_equal(bits(z), bits(np.concatenate([p[3] for p in parts], axis=1)))
    else:
        assert z is None


def test_gemv_on_concatenated_qkv():
    """Llama-3-8B q, k, v (4096 + 1024 + 1024 rows, K = 4096) as one GEMV: every
    output equals the oracle's product with the concatenated W'."""
    K = 4096
    parts = [oracle_layer(n, K, 0.02, 0.0, True, i) for i, n in enumerate((4096, 1024, 1024))]
    q, s, z = awq.awq_concat_rows([(dev(p[1]), dev(p[2]), dev(p[3])) for p in parts])
    Wd = np.concatenate([p[4] for p in parts], axis=0)
    for M in (1, 5):
        x = activations(M, K, seed=90 + M)
        ws = awq.alloc_workspace(M, 6144, K, True)
        y = host(awq.awq_gemv(dev(x), q, s, z, workspace=ws))
        assert_close(y, O.matmul_f64(x, Wd), f"qkv M={M}")
