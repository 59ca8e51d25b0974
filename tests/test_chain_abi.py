"""Host-side checks of awq_gemv_chain through the C ABI (no GPU): every call
below fails validation before the library touches the CUDA runtime, so the
fake device addresses are never dereferenced."""

import ctypes

import pytest

import weight_only_int4_gemv_b200 as awq

OK, NULL, SHAPE, ALIGN, UNSUP, CUDA, WS = range(7)
A = 0x10000


@pytest.fixture(scope="module")
def L():
    import os
    if not os.path.exists(awq.LIB_PATH):
        from weight_only_int4_gemv_b200 import build
        build.build()
    return awq.lib()


def layer(x=A, q=A + 0x1000, s=A + 0x2000, z=A + 0x3000, y=A + 0x4000, N=64, K=256, zp=1, flags=0, x_from=-1):
    return awq.GemvLayer(x, q, s, z if zp else None, y, N, K, awq.QConfig(128, zp, flags), x_from)


def call(L, layers, M=1, n=None):
    arr = (awq.GemvLayer * max(1, len(layers)))(*layers)
    nb = ctypes.c_size_t(0)
    return L.awq_gemv_chain_workspace_bytes(arr, len(layers) if n is None else n, M, ctypes.byref(nb))


def test_chain_symbols_and_struct(L):
    assert hasattr(L, "awq_gemv_chain") and hasattr(L, "awq_gemv_chain_workspace_bytes")
    assert hasattr(L, "awq_debug_set_wait_limit_ns")
    # awq_gemv_layer_t: five pointers, two int64, the 12-byte config, an int32
    assert ctypes.sizeof(awq.GemvLayer) == 72


def test_chain_counts_and_batch(L):
    assert L.awq_gemv_chain_workspace_bytes(None, 1, 1, ctypes.byref(ctypes.c_size_t())) == NULL
    assert call(L, [layer()], n=0) == SHAPE
    assert call(L, [layer()] * 33) == SHAPE                # more than AWQ_CHAIN_MAX_LAYERS
    assert call(L, [layer()], M=0) == SHAPE
    assert call(L, [layer()], M=17) == SHAPE
    arr = (awq.GemvLayer * 1)(layer())
    assert L.awq_gemv_chain_workspace_bytes(arr, 1, 1, None) == NULL


def test_chain_layer_checks(L):
    assert call(L, [layer(N=60)]) == SHAPE                 # N % 8
    assert call(L, [layer(N=0)]) == SHAPE
    assert call(L, [layer(K=200)]) == SHAPE                # K % 128
    assert call(L, [layer(x=0)]) == NULL
    assert call(L, [layer(zp=1, z=0)]) == NULL             # asymmetric without zeros
    assert call(L, [layer(x=A + 2)]) == ALIGN
    assert call(L, [layer(flags=awq.FLAG_SILU_MUL, N=48)]) == SHAPE
    assert call(L, [layer(flags=8)]) == UNSUP              # undefined flag
    # one zero-point form per call
    assert call(L, [layer(zp=1), layer(zp=0, x=A + 0x8000, y=A + 0x9000)]) == UNSUP


def test_chain_dependency_checks(L):
    l0 = layer(N=256, K=256)
    # x_from must name an earlier layer
    assert call(L, [layer(x_from=0)]) == SHAPE
    assert call(L, [l0, layer(x_from=1, x=A + 0x4000)]) == SHAPE
    assert call(L, [l0, layer(x_from=-2)]) == SHAPE
    # x must be that layer's y, and K its column count
    assert call(L, [l0, layer(x_from=0, x=A + 0x5000, K=256)]) == SHAPE
    assert call(L, [l0, layer(x_from=0, x=A + 0x4000, K=384)]) == SHAPE
    # with the fused gate/up epilogue the source has N/2 columns
    g = layer(N=512, K=256, flags=awq.FLAG_SILU_MUL)
    assert call(L, [g, layer(x_from=0, x=A + 0x4000, K=512)]) == SHAPE
