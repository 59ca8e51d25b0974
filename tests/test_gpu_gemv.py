"""GPU parity of awq_gemv (1 <= M <= 16) against the float64 oracle.

Weights come from the seeded generator and are quantized by the oracle, so
the only difference between the two sides is the CUDA kernel's arithmetic.
Full-size Llama-shaped layers are compared on every output; the 70B shapes on
sampled output channels (their oracle quantization is checked bit-exact on
the same rows)."""

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import (activations, assert_close, bits, dev, host, oracle_layer, sample_rows)
from workloads import make_layer, make_packed_random, make_weight

pytestmark = pytest.mark.gpu


def run_gemv(x, qweight, scales, zeros, weights_static=False):
    M, K = x.shape
    N = qweight.shape[0]
    ws = awq.alloc_workspace(M, N, K, zeros is not None)
    y = awq.awq_gemv(dev(x), dev(qweight), dev(scales), dev(zeros) if zeros is not None else None,
                     workspace=ws, weights_static=weights_static)
    torch.cuda.synchronize()
    return host(y), ws


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(512, 512), (8, 128), (40, 256), (1000, 1024), (4096, 4096)])
def test_gemv_small_shapes_all_batches(N, K, zp):
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, zp)
    for M in range(1, 17):
        x = activations(M, K, seed=M)
        y, _ = run_gemv(x, qweight, scales, zeros)
        assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M} zp={zp}")


def test_gemv_single_512_layer():
    """The 512 x 512 parity layer: W ~ N(0, 0.02), asym g128, x[1, 512], seed 0."""
    W, x = make_layer(512, 512, 1, 0.02, 0.0, seed=0)
    codes, scales, zeros = O.pseudo_quantize(W, 128, True)
    y, _ = run_gemv(x, O.pack(codes), scales, zeros)
    assert_close(y, O.matmul_f64(x, O.dequant(codes, scales, zeros, 128)), "512x512")


@pytest.mark.parametrize("name,N,K", [("q_proj", 4096, 4096), ("gate_up_proj", 14336, 4096),
                                      ("down_proj", 4096, 14336)])
def test_gemv_llama3_8b_decode_m1(name, N, K):
    """Llama-3-8B decode layers at M = 1 with 1% salient input channels x10."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(1, K, seed=1)
    y, _ = run_gemv(x, qweight, scales, zeros)
    assert_close(y, O.matmul_f64(x, Wd), name)


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("N,K", [(14336, 4096), (4096, 14336)])
def test_gemv_decode_sweep(N, K, zp):
    """M in {1, 2, 4, 8, 16}, asymmetric and symmetric."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.0, zp)
    for M in (1, 2, 4, 8, 16):
        x = activations(M, K, seed=10 + M)
        y, _ = run_gemv(x, qweight, scales, zeros)
        assert_close(y, O.matmul_f64(x, Wd), f"N={N} K={K} M={M} zp={zp}")


@pytest.mark.parametrize("N,K", [(8192, 8192), (28672, 8192), (8192, 28672)])
def test_gemv_llama3_70b_sampled(N, K):
    """70B shapes at M in {1, 8}: GPU-quantized weights, oracle on sampled rows."""
    W = make_weight(N, K, 0.015, 0.01, seed=0)
    qg, sg, zg = awq.awq_pseudo_quantize_pack(dev(W), zero_point=True)
    rows = sample_rows(N, 256)
    codes, scales, zeros = O.pseudo_quantize(W[rows], 128, True)
    assert np.array_equal(bits(host(qg)[rows]), bits(O.pack(codes)))
    Wd = O.dequant(codes, scales, zeros, 128)
    for M in (1, 8):
        x = activations(M, K, seed=20 + M)
        ws = awq.alloc_workspace(M, N, K, True)
        y = host(awq.awq_gemv(dev(x), qg, sg, zg, workspace=ws))
        assert_close(y[:, rows], O.matmul_f64(x, Wd), f"N={N} K={K} M={M}")


def test_gemv_random_codes_and_extreme_zero_points():
    """Arbitrary words (every code value in every slot) and zero points 0..15."""
    for zp in (True, False):
        qweight, scales, zeros = make_packed_random(296, 2048, 128, zp, seed=4)
        Wd = O.dequant(O.unpack(qweight), scales, zeros, 128)
        for M in (1, 5, 16):
            x = activations(M, 2048, seed=M)
            y, _ = run_gemv(x, qweight, scales, zeros)
            assert_close(y, O.matmul_f64(x, Wd), f"random zp={zp} M={M}")


def test_gemv_is_deterministic_and_reuses_its_workspace():
    """Repeated calls on one workspace give identical bits and stay correct.
    N = 1024 has fewer 16-channel tiles than the GPU has SMs, so K is cut
    into slices that different CTAs sum; a tile is finished only when its
    arrival counter reaches the slice count, so a counter left non-zero would
    leave tiles unfinished."""
    _, qweight, scales, zeros, Wd = oracle_layer(1024, 14336, 0.02, 0.0, True)
    x = activations(4, 14336, seed=3)
    ws = awq.alloc_workspace(4, 1024, 14336, True)
    assert ws is not None
    ys = []
    for _ in range(4):
        y = torch.full((4, 1024), float("nan"), dtype=torch.float16, device="cuda")
        awq.awq_gemv(dev(x), dev(qweight), dev(scales), dev(zeros), workspace=ws, out=y)
        torch.cuda.synchronize()
        ys.append(bits(y))
    for yb in ys[1:]:
        assert np.array_equal(ys[0], yb)
    assert_close(ys[-1].view(np.float16), O.matmul_f64(x, Wd), "4th call")


@pytest.mark.parametrize("M,N,K", [(1, 14336, 4096), (3, 4096, 14336), (16, 1000, 2048)])
def test_gemv_repeated_calls_give_identical_bits(M, N, K):
    """Partial sums meet in a fixed order (inside a CTA and across K
    slices), so repeated calls agree bit for bit."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, True)
    x = activations(M, K, seed=4)
    ys = [bits(run_gemv(x, qweight, scales, zeros)[0]) for _ in range(3)]
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])
    assert_close(ys[0].view(np.float16), O.matmul_f64(x, Wd), f"M={M} N={N} K={K}")


def test_gemv_whole_tiles_need_no_workspace():
    """With at least one 16-channel tile per CTA (two CTAs per SM for M <= 8)
    every CTA covers all of K for its tiles: no workspace, and the call works
    without one."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    for M, N, K in [(1, 32 * sms, 4096), (8, 32 * sms, 1024), (16, 14336, 4096), (12, 16 * sms, 4096)]:
        assert awq.awq_workspace_bytes(M, N, K, True) == 0, (M, N, K)
    _, qweight, scales, zeros, Wd = oracle_layer(32 * sms, 1024, 0.02, 0.01, True)
    x = activations(2, 1024, seed=7)
    y = host(awq.awq_gemv(dev(x), dev(qweight), dev(scales), dev(zeros), workspace=None))
    assert_close(y, O.matmul_f64(x, Wd), "N = 32 x SMs")


@pytest.mark.parametrize("zp", [True, False])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (1, 14336, 4096), (8, 4096, 14336), (16, 1000, 2048),
                                   (3, 40, 256), (1, 2360, 1024)])
def test_gemv_weights_static_gives_the_same_bits(M, N, K, zp):
    """AWQ_FLAG_WEIGHTS_STATIC only moves when the weights are read (before
    the previous kernel on the stream completes), never what is computed."""
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, zp)
    x = activations(M, K, seed=5)
    y0, _ = run_gemv(x, qweight, scales, zeros)
    y1, _ = run_gemv(x, qweight, scales, zeros, weights_static=True)
    assert np.array_equal(bits(y0), bits(y1))
    assert_close(y1, O.matmul_f64(x, Wd), f"static M={M} N={N} K={K}")


def test_gemv_back_to_back_layers_weights_static():
    """A chain of dependent layers on one stream with the flag set: each
    layer's x is the previous layer's y, written by the kernel just before."""
    layers = [oracle_layer(1024, 1024, 0.02, 0.01, True, seed=s) for s in range(4)]
    x0 = activations(2, 1024, seed=9)
    xs = [dev(x0)]
    for (_, q, s, z, _) in layers:
        y = awq.awq_gemv(xs[-1], dev(q), dev(s), dev(z), workspace=awq.alloc_workspace(2, 1024, 1024, True),
                         weights_static=True)
        xs.append(y)
    torch.cuda.synchronize()
    xr = x0
    for i, (_, _, _, _, Wd) in enumerate(layers):
        yr = O.matmul_f64(xr, Wd)
        assert_close(host(xs[i + 1]), yr, f"layer {i}")
        xr = yr.astype(np.float16)     # the oracle's own fp16 output feeds its next layer


def test_gemv_workspace_required_and_checked():
    _, qweight, scales, zeros, _ = oracle_layer(1024, 4096, 0.02, 0.01, True)
    x = dev(activations(2, 4096))
    need = awq.awq_workspace_bytes(2, 1024, 4096, True)
    assert need > 0
    small = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(awq.AwqError, match="WORKSPACE"):
        awq.awq_gemv(x, dev(qweight), dev(scales), dev(zeros), workspace=small)
    with pytest.raises(awq.AwqError, match="WORKSPACE"):
        awq.awq_gemv(x, dev(qweight), dev(scales), dev(zeros), workspace=None)


def test_gemv_edge_cases():
    _, qweight, scales, zeros, _ = oracle_layer(512, 512, 0.02, 0.01, True)
    # M out of range
    with pytest.raises(awq.AwqError, match="SHAPE"):
        awq.awq_gemv(dev(activations(17, 512)), dev(qweight), dev(scales), dev(zeros))
    # N must be a multiple of 8 (16-byte runs of scales and zero points)
    q2, s2, z2 = make_packed_random(300, 512, 128, True, seed=1)
    with pytest.raises(awq.AwqError, match="SHAPE"):
        awq.awq_gemv(dev(activations(1, 512)), dev(q2), dev(s2), dev(z2))
    # unsupported group size
    with pytest.raises(awq.AwqError, match="UNSUPPORTED"):
        awq.awq_gemv(dev(activations(1, 512)), dev(qweight), dev(scales), dev(zeros), group_size=64)
    # misaligned output
    buf = torch.zeros(512 + 8, dtype=torch.float16, device="cuda")
    y_bad = buf[1:513].view(1, 512)
    ws = awq.alloc_workspace(1, 512, 512, True)
    with pytest.raises(awq.AwqError, match="ALIGN"):
        awq.awq_gemv(dev(activations(1, 512)), dev(qweight), dev(scales), dev(zeros), workspace=ws, out=y_bad)
    # empty weight matrix: nothing to do
    y = awq.awq_gemv(dev(activations(3, 256)), torch.empty((0, 32), dtype=torch.int32, device="cuda"),
                     torch.empty((2, 0), dtype=torch.float16, device="cuda"),
                     torch.empty((2, 0), dtype=torch.float16, device="cuda"))
    assert y.shape == (3, 0)
