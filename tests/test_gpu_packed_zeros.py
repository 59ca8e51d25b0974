"""GPU parity of the packed zero points (AWQ_FLAG_PACKED_ZEROS, int32 qzeros
[G][N/8]): awq_pack_zeros / awq_unpack_zeros bit for bit against the oracle,
awq_dequant with packed zero points bit for bit against the oracle's
dequantization, and awq_gemv and awq_gemm with packed zero points against
the float64 oracle and bit for bit against the same call with the fp16 zero
points."""

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


@pytest.mark.parametrize("G,N", [(1, 8), (3, 24), (32, 4096), (112, 4096), (5, 1000)])
def test_pack_zeros_matches_the_oracle(G, N):
    rng = np.random.default_rng(G * 7 + N)
    z = rng.integers(0, 16, size=(G, N)).astype(np.float16)
    q = awq.awq_pack_zeros(dev(z))
    torch.cuda.synchronize()
    assert q.dtype == torch.int32 and tuple(q.shape) == (G, N // 8)
    assert np.array_equal(bits(q), bits(O.pack_zeros(z)))
    back = awq.awq_unpack_zeros(q)
    torch.cuda.synchronize()
    assert np.array_equal(bits(back), bits(z))


def test_pack_zeros_rounds_and_clamps_like_the_oracle():
    # non-integers (ties to even), out-of-range values, infinities and NaN
    vals = np.array([2.5, 3.5, -1.0, 17.0, np.nan, np.inf, -np.inf, 14.6, 0.49, 7.5, -0.0, 15.0,
                     1e-7, 65504.0, -65504.0, 8.5], dtype=np.float16)
    z = np.tile(vals, (4, 4))
    q = awq.awq_pack_zeros(dev(z))
    torch.cuda.synchronize()
    assert np.array_equal(bits(q), bits(O.pack_zeros(z)))


def test_unpack_zeros_matches_the_oracle():
    rng = np.random.default_rng(21)
    words = rng.integers(0, 2 ** 32, size=(7, 40), dtype=np.uint64).astype(np.uint32).view(np.int32)
    z = awq.awq_unpack_zeros(dev(words))
    torch.cuda.synchronize()
    assert np.array_equal(bits(z), bits(O.unpack_zeros(words)))


@pytest.mark.parametrize("N,K", [(8, 128), (40, 256), (4096, 512), (1000, 1024)])
def test_dequant_with_packed_zeros_is_bit_exact(N, K):
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    qz = O.pack_zeros(zeros)
    Wg = awq.awq_dequant(dev(qweight), dev(scales), dev(qz))
    torch.cuda.synchronize()
    assert np.array_equal(bits(Wg), bits(Wd))


def _gemv_pair(M, N, K, seed=5, weights_static=False):
    """(y with fp16 zero points, y with packed zero points, x, W')."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(M, K, seed=seed)
    ws = awq.alloc_workspace(M, N, K, True)
    q, s = dev(qweight), dev(scales)
    y16 = awq.awq_gemv(dev(x), q, s, dev(zeros), workspace=ws, weights_static=weights_static)
    y4 = awq.awq_gemv(dev(x), q, s, dev(O.pack_zeros(zeros)), workspace=ws, weights_static=weights_static)
    torch.cuda.synchronize()
    return host(y16), host(y4), x, Wd


@pytest.mark.parametrize("N,K", [(32, 128), (96, 256), (1056, 1024), (4096, 512), (2080, 2048)])
def test_gemv_packed_zeros_small_shapes_all_batches(N, K):
    """Shapes with few tiles (K slices meet in the workspace), a ragged last
    64-row block (N = 1056, 2080) and chunks that start on odd tiles."""
    for M in (1, 2, 3, 8, 9, 16):
        y16, y4, x, Wd = _gemv_pair(M, N, K, seed=M)
        assert np.array_equal(bits(y4), bits(y16)), f"M={M}"
        assert_close(y4, O.matmul_f64(x, Wd), f"packed M={M} N={N} K={K}")


@pytest.mark.parametrize("N,K", [(4096, 4096), (14336, 4096), (4096, 14336)])
def test_gemv_packed_zeros_llama3_8b_shapes(N, K):
    """The decode shapes: bit-identical to the fp16 zero points at M = 1 and
    4 (the fp16 path is checked against the oracle at these sizes), and
    sampled rows against the float64 oracle."""
    rows = sample_rows(N, 256)
    for M in (1, 4):
        y16, y4, x, Wd = _gemv_pair(M, N, K, seed=10 + M, weights_static=True)
        assert np.array_equal(bits(y4), bits(y16)), f"M={M}"
        assert_close(y4[:, rows], O.matmul_f64(x, Wd[rows]), f"packed M={M} N={N} K={K}")


def test_gemv_packed_zeros_noalloc_and_fused_gate_up():
    N, K = 512, 1024
    # awq_gemv_noalloc with packed zero points
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(3, K, seed=4)
    y = awq.awq_gemv_noalloc(dev(x), dev(qweight), dev(scales), dev(O.pack_zeros(zeros)))
    torch.cuda.synchronize()
    assert_close(host(y), O.matmul_f64(x, Wd), "noalloc packed")
    # the fused gate/up layout: its fp16 zero points interleaved, then packed
    _, qg, sg, zg, Wg = oracle_layer(N, K, 0.02, 0.0, True, 0)
    _, qu, su, zu, Wu = oracle_layer(N, K, 0.02, 0.0, True, 1)
    q, s, z = awq.awq_interleave_gate_up(dev(qg), dev(sg), dev(zg), dev(qu), dev(su), dev(zu))
    qz = awq.awq_pack_zeros(z)
    for M in (1, 5, 16):
        xm = activations(M, K, seed=20 + M)
        ws = awq.alloc_workspace(M, 2 * N, K, True, silu_mul=True)
        h16 = awq.awq_gemv(dev(xm), q, s, z, workspace=ws, silu_mul=True)
        h4 = awq.awq_gemv(dev(xm), q, s, qz, workspace=ws, silu_mul=True)
        torch.cuda.synchronize()
        assert np.array_equal(bits(h4), bits(h16)), f"M={M}"
        assert_close(host(h4), O.gate_up_silu_f64(xm, Wg, Wu), f"fused packed M={M}")


@pytest.mark.parametrize("M,N,K,silu", [(17, 256, 512, False), (128, 4096, 4096, False), (300, 1024, 2048, False),
                                       (2048, 512, 1024, False), (96, 2048, 1024, True)])
def test_gemm_with_packed_zeros_matches_fp16_zeros(M, N, K, silu):
    """awq_gemm with int32 qzeros (unpacked into the workspace by the call)
    gives the bits of the same call with the fp16 zero points, and stays
    within the oracle's tolerance; with the fused gate/up layout too."""
    if silu:
        half = N // 2
        _, qg, sg, zg, Wg = oracle_layer(half, K, 0.02, 0.01, True, seed=41)
        _, qu, su, zu, Wu = oracle_layer(half, K, 0.02, 0.01, True, seed=42)
        q, s, z = awq.awq_interleave_gate_up(dev(qg), dev(sg), dev(zg), dev(qu), dev(su), dev(zu))
    else:
        _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True, seed=M)
        q, s, z = dev(qweight), dev(scales), dev(zeros)
    qz = awq.awq_pack_zeros(z)
    xh = activations(M, K, seed=M + 1)
    x = dev(xh)
    ws16 = awq.alloc_workspace(M, N, K, True, silu_mul=silu)
    ws4 = awq.alloc_workspace(M, N, K, True, silu_mul=silu, packed_zeros=True)
    assert ws4 is not None and ws4.numel() >= (K // 128) * N * 2
    y16 = awq.awq_gemm(x, q, s, z, workspace=ws16, silu_mul=silu)
    y4 = awq.awq_gemm(x, q, s, qz, workspace=ws4, silu_mul=silu)
    torch.cuda.synchronize()
    assert np.array_equal(bits(y4), bits(y16))
    if silu:
        assert_close(host(y4), O.gate_up_silu_f64(xh, Wg, Wu), f"fused packed gemm M={M}")
    else:
        rows = sample_rows(N, 512, seed=M)
        assert_close(host(y4)[:, rows], O.matmul_f64(xh, Wd[rows]), f"packed gemm M={M}")
    # awq_linear takes either form at any M
    yl = awq.awq_linear(x, q, s, qz, workspace=ws4, silu_mul=silu)
    torch.cuda.synchronize()
    assert np.array_equal(bits(yl), bits(y16))


def test_gemm_packed_zeros_without_room_is_refused():
    _, qweight, scales, zeros, _ = oracle_layer(256, 512, 0.02, 0.01, True)
    x = dev(activations(32, 512))
    with pytest.raises(awq.AwqError, match="WORKSPACE"):
        awq.awq_gemm(x, dev(qweight), dev(scales), dev(O.pack_zeros(zeros)))
