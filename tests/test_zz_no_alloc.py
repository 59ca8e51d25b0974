"""awq_gemv_noalloc: the GEMV entry point that allocates nothing.

Some callers of this library cannot allocate device memory when they run the
layer: a plugin inside a host engine that owns all device memory and hands in
only the input and output buffers, or a decode loop that must not allocate
after start-up. awq_gemv_noalloc serves them from one fixed scratch array
inside the library instead of a caller workspace. These tests call it through
the C ABI and check it against awq_gemv with a caller workspace, on two calls
in a row (the array keeps the previous call's contents). The file is named
so that pytest collects it after every other test file.
"""

import ctypes
import os
import re

import numpy as np
import pytest
import torch

import weight_only_int4_gemv_b200 as awq
from oracle import awq_oracle as O
from parity_util import activations, assert_close, bits, dev, host, oracle_layer


def test_noalloc_is_exported_and_validates_on_the_host():
    L = awq.lib()
    assert hasattr(L, "awq_gemv_noalloc")
    P, A = ctypes.c_void_p, 0x10000
    cfg = awq.QConfig(128, 1)
    # rejected before any CUDA call: null input, batch out of range, N % 8, group size
    assert L.awq_gemv_noalloc(None, P(A), P(A), P(A), 1, 64, 256, cfg, P(A), None) == 1
    assert L.awq_gemv_noalloc(P(A), P(A), P(A), P(A), 17, 64, 256, cfg, P(A), None) == 2
    assert L.awq_gemv_noalloc(P(A), P(A), P(A), P(A), 1, 60, 256, cfg, P(A), None) == 2
    assert L.awq_gemv_noalloc(P(A), P(A), P(A), P(A), 1, 64, 256, awq.QConfig(64, 1), P(A), None) == 4


@pytest.mark.gpu
@pytest.mark.parametrize("M,N,K,zp", [(1, 14336, 4096, True), (4, 4096, 14336, True),
                                      (16, 4096, 4096, False), (3, 1000, 1024, True)])
def test_noalloc_matches_workspace_entry_on_two_calls(M, N, K, zp):
    _, qweight, scales, zeros, Wd = oracle_layer(N, K, 0.02, 0.01, zp)
    xh = activations(M, K, seed=M)
    x, q, s = dev(xh), dev(qweight), dev(scales)
    z = dev(zeros) if zp else None
    ws = awq.alloc_workspace(M, N, K, zp)
    ref = host(awq.awq_gemv(x, q, s, z, workspace=ws))
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        awq.awq_gemv_noalloc(x, q, s, z, out=y)
        torch.cuda.synchronize()
        yh = host(y)
        # the parity tolerance of the other tests, against the existing entry point
        assert_close(yh, ref.astype(np.float64), f"call {call} vs awq_gemv")
        # same kernel and same split: the bits agree too
        assert np.array_equal(bits(yh), bits(ref)), f"call {call}"
    assert_close(yh, O.matmul_f64(xh, Wd), "vs oracle")


@pytest.mark.gpu
def test_noalloc_array_covers_every_shape():
    """Only shapes with fewer 16-channel tiles than SMs use scratch (K slices
    summed across CTAs), and their need is bounded by about two items per SM:
    the fixed array holds it for every batch size and K. A shape whose need
    exceeded the array would be refused with AWQ_ERR_WORKSPACE before any
    device work."""
    header = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "awq.h")).read()
    m = re.search(r"#define AWQ_GEMV_STATIC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", header)
    cap = int(m.group(1)) << int(m.group(2))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    worst = 0
    for M in (1, 8, 9, 16):
        for N in (8, 16, 120, 1000, 16 * sms - 8, 16 * sms, 4096, 28672):
            for K in (128, 4096, 28672, 1 << 20):
                worst = max(worst, awq.awq_workspace_bytes(M, N, K, True))
                worst = max(worst, awq.awq_workspace_bytes(M, N, K, False))
                if N % 32 == 0:
                    # the fused gate/up layout (units of two tiles) and packed zero points
                    for silu, packed in [(True, False), (False, True), (True, True)]:
                        worst = max(worst, awq.awq_workspace_bytes(M, N, K, True, silu_mul=silu,
                                                                   packed_zeros=packed))
    assert 0 < worst <= cap


@pytest.mark.gpu
@pytest.mark.parametrize("M,packed", [(1, False), (8, True), (16, True)])
def test_noalloc_fused_gate_up_and_packed_zeros(M, packed):
    """The fused SiLU epilogue and packed zero points through the fixed array:
    gate + up of 512 rows each (2N = 1024, fewer tiles than SMs, so K is split
    across CTAs and the partials go through the array), bit for bit against
    awq_gemv with a caller workspace on two calls in a row."""
    N, K = 512, 4096
    _, qg, sg, zg, _ = oracle_layer(N, K, 0.02, 0.01, True, seed=11)
    _, qu, su, zu, _ = oracle_layer(N, K, 0.02, 0.01, True, seed=12)
    q, s, z = awq.awq_interleave_gate_up(dev(qg), dev(sg), dev(zg), dev(qu), dev(su), dev(zu))
    if packed:
        z = awq.awq_pack_zeros(z)
    x = dev(activations(M, K, seed=3))
    ws = awq.alloc_workspace(M, 2 * N, K, True, silu_mul=True, packed_zeros=packed)
    assert ws is not None      # the shape does split K
    ref = host(awq.awq_gemv(x, q, s, z, workspace=ws, silu_mul=True))
    torch.cuda.synchronize()
    for call in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float16, device="cuda")
        awq.awq_gemv_noalloc(x, q, s, z, out=y, silu_mul=True)
        torch.cuda.synchronize()
        assert np.array_equal(bits(host(y)), bits(ref)), f"call {call}"
