"""Pins of the oracle's packed zero points (qzeros) against hand-worked words,
the nibble arithmetic, round trips and the dequantization they feed."""
import os

import numpy as np

from oracle import awq_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_packed_zeros_golden_words():
    for r in _rows("packed_zeros_words.txt"):
        z = np.array([[float(v) for v in r[:8]]], dtype=np.float16)
        w = O.pack_zeros(z)
        assert w.dtype == np.int32 and w.shape == (1, 1)
        assert int(w.view(np.uint32)[0, 0]) == int(r[8], 16)
        assert np.array_equal(O.unpack_zeros(w), z)


def test_packed_zeros_every_slot_every_value():
    # channel n of a word sits at bits 4n .. 4n+3, nothing else is set
    for n in range(8):
        for v in range(16):
            z = np.zeros((1, 8), dtype=np.float16)
            z[0, n] = v
            assert int(O.pack_zeros(z).view(np.uint32)[0, 0]) == v * 16 ** n


def test_packed_zeros_axis_and_group_rows():
    # word w of group row j holds channels 8w..8w+7 of that group only
    G, N = 3, 24
    z = np.zeros((G, N), dtype=np.float16)
    z[2, 13] = 9          # group 2, word 1, nibble 5
    w = O.pack_zeros(z).view(np.uint32)
    assert w.shape == (G, N // 8)
    expect = np.zeros((G, N // 8), dtype=np.uint32)
    expect[2, 1] = 9 << 20
    assert np.array_equal(w, expect)


def test_packed_zeros_roundtrip():
    rng = np.random.default_rng(11)
    z = rng.integers(0, 16, size=(32, 4096)).astype(np.float16)
    assert np.array_equal(O.unpack_zeros(O.pack_zeros(z)), z)
    words = rng.integers(0, 2 ** 32, size=(4, 64), dtype=np.uint64).astype(np.uint32).view(np.int32)
    assert np.array_equal(O.pack_zeros(O.unpack_zeros(words)), words)


def test_packed_zeros_out_of_range_values():
    # nearest integer (ties to even), clamped to 0..15, NaN -> 0
    z = np.array([[2.5, 3.5, -1.0, 17.0, np.nan, np.inf, -np.inf, 14.6]], dtype=np.float16)
    got = O.unpack_zeros(O.pack_zeros(z)).astype(np.float64)[0]
    assert list(got) == [2, 4, 0, 15, 0, 15, 0, 15]


def test_dequant_with_unpacked_zeros_is_unchanged():
    # the zero points the quantizer writes survive packing, so the weights do too
    rng = np.random.default_rng(12)
    W = (rng.standard_normal((64, 512)) * 0.02).astype(np.float16)
    codes, s, z = O.pseudo_quantize(W, zero_point=True)
    z2 = O.unpack_zeros(O.pack_zeros(z))
    assert np.array_equal(z2, z)
    a = O.dequant(codes, s, z).view(np.uint16)
    b = O.dequant(codes, s, z2).view(np.uint16)
    assert np.array_equal(a, b)


def test_packed_zeros_byte_arithmetic():
    # 4-bit codes + fp16 scale + 4-bit zero point per group of 128 weights
    N, K = 4096, 4096
    G = K // O.GROUP_SIZE
    codes, scales, qzeros = N * K // 2, 2 * G * N, G * N // 2
    assert qzeros == O.pack_zeros(np.zeros((G, N), np.float16)).nbytes
    bits = 8 * (codes + scales + qzeros) / (N * K)
    assert abs(bits - (4 + 16 / 128 + 4 / 128)) < 1e-12      # 4.156 bits per weight (4.25 with fp16 zeros)
