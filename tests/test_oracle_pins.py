"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test checks the oracle against something the pages or mathematics fix:
hand-worked examples (tests/golden, each citing its page and section),
closed forms evaluated with an fp16 rounding written here from the IEEE
definition (not numpy's cast), brute-force argmin searches on small groups,
exact integer arithmetic, and the scale-migration invariant of the AutoAWQ
tour ("The big picture"). A plausible slip in the oracle (a dropped zero
point, a wrong sign, a transposed operand, a wrong nibble slot, the wrong
rounding mode) fails at least one of them.
"""

import os
import warnings
from fractions import Fraction

import numpy as np
import pytest

from oracle import awq_oracle as O
from workloads import make_layer, make_packed_random, make_weight

# ----------------------------------------------------------------------------
# fp16 from first principles: value of every positive bit pattern by the
# IEEE binary16 formula, and nearest-even rounding by table search.
# ----------------------------------------------------------------------------
_BITS = np.arange(0x7C01, dtype=np.int64)          # +0 .. +inf
_EXP = (_BITS >> 10) & 0x1F
_MAN = _BITS & 0x3FF
_VALS = np.where(_EXP == 0, np.ldexp(_MAN.astype(np.float64), -24),
                 np.ldexp((1024 + _MAN).astype(np.float64), (_EXP - 25).astype(np.int64)))
_VALS[0x7C00] = 65536.0                             # rounding slot standing for +inf


def f16_bits_nearest(v):
    """fp16 bit patterns of float64 values, round to nearest, ties to even."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    i = np.clip(np.searchsorted(_VALS, a, side="left"), 1, len(_VALS) - 1)
    lo, hi = i - 1, i
    dlo = a - _VALS[lo]
    dhi = _VALS[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (_BITS[hi] % 2 == 0))
    bits = np.where(pick_hi, _BITS[hi], _BITS[lo])
    bits = np.where(a == 0, 0, bits)
    bits = np.where(a >= 65536.0, 0x7C00, bits)      # overflow to inf
    sign = np.where(np.signbit(v), 0x8000, 0)
    return (bits | sign).astype(np.uint16)


def f16_value(bits):
    """float64 value of fp16 bit patterns (finite), from the IEEE formula."""
    b = np.asarray(bits, dtype=np.int64)
    mag = _VALS[b & 0x7FFF]
    return np.where(b & 0x8000, -mag, mag)


def bits16(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def _read_golden(golden_dir, name):
    rows = []
    with open(os.path.join(golden_dir, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


# ----------------------------------------------------------------------------
# the fp16 helper itself
# ----------------------------------------------------------------------------
def test_fp16_helper_known_values():
    assert f16_bits_nearest([1.0])[0] == 0x3C00
    assert f16_bits_nearest([65504.0])[0] == 0x7BFF
    assert f16_bits_nearest([2.0 ** -24])[0] == 0x0001
    assert f16_bits_nearest([-2.0])[0] == 0xC000
    assert f16_bits_nearest([1.0 + 2.0 ** -11])[0] == 0x3C00        # tie -> even
    assert f16_bits_nearest([1.0 + 3 * 2.0 ** -11])[0] == 0x3C02    # tie -> even
    assert f16_bits_nearest([65520.0])[0] == 0x7C00                 # tie at max -> inf
    assert f16_bits_nearest([2.0 ** -26])[0] == 0x0000              # below half of min subnormal
    # every finite fp16 value maps to its own pattern
    pos = np.arange(0x7C00)
    assert np.array_equal(f16_bits_nearest(_VALS[pos]), pos.astype(np.uint16))


# ----------------------------------------------------------------------------
# dequant: closed form (AutoAWQ tour zero-point decode; fak "Dequantization
# Formula" for the symmetric decode)
# ----------------------------------------------------------------------------
def _scale_sweep():
    pats = np.unique(np.concatenate([
        np.arange(1, 0x7C00, 7), [0x0001, 0x00A8, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x211F]]))
    return pats.astype(np.uint16)


@pytest.mark.parametrize("z", list(range(16)) + [None])
def test_dequant_closed_form_exhaustive(z):
    sbits = _scale_sweep()
    S = len(sbits)
    codes = np.tile(np.tile(np.arange(16, dtype=np.uint8), 8), (S, 1))      # [S, 128]
    scales = sbits.view(np.float16).reshape(1, S)                           # [G=1, N=S]
    zeros = None if z is None else np.full((1, S), z, dtype=np.float16)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        got = bits16(O.dequant(codes, scales, zeros, 128))
    zz = 8 if z is None else z
    exact = (codes.astype(np.float64) - zz) * f16_value(sbits).reshape(S, 1)   # exact in f64
    assert np.array_equal(got, f16_bits_nearest(exact))


def test_sym_dequant_golden(golden_dir):
    rows = _read_golden(golden_dir, "sym_dequant_scale_0x211f.txt")
    sbits = int(rows[0][1], 16)
    table = {int(r[0]): int(r[1], 16) for r in rows[1:]}
    codes = np.tile(np.array(sorted(table), dtype=np.uint8), 8).reshape(1, 128)
    scales = np.array([[sbits]], dtype=np.uint16).view(np.float16)
    got = bits16(O.dequant(codes, scales, None, 128))[0, :16]
    assert [int(b) for b in got] == [table[c] for c in sorted(table)]


# ----------------------------------------------------------------------------
# quantize: hand-worked examples
# ----------------------------------------------------------------------------
def test_asym_group_golden(golden_dir):
    rows = {r[0]: r[1:] for r in _read_golden(golden_dir, "asym_group_worked.txt")}
    vals = [float(v) for v in rows["values"]]
    w = np.zeros((1, 128), dtype=np.float16)
    w[0, :len(vals)] = np.array(vals, dtype=np.float16)
    codes, scales, zeros = O.quantize_asym(w, 128)
    assert float(scales[0, 0]) == float(rows["scale"][0])
    assert float(zeros[0, 0]) == float(rows["zero"][0])
    assert codes[0, :len(vals)].tolist() == [int(c) for c in rows["codes"]]
    assert np.all(codes[0, len(vals):] == int(rows["rest_code"][0]))
    deq = O.dequant(codes, scales, zeros, 128)
    assert deq[0, :len(vals)].astype(np.float64).tolist() == [float(v) for v in rows["dequant"]]


def test_zero_points_are_positive_integers():
    """Zero points are the integers 0..15 stored as fp16, zero as +0 (an
    all-positive group has -rint(min/s) = -0)."""
    W = np.abs(np.random.default_rng(11).normal(0, 0.02, (8, 256))).astype(np.float16)
    _, _, zeros = O.quantize_asym(W, 128)
    zb = bits16(zeros)
    assert np.all(zb == 0)
    W2 = np.random.default_rng(12).normal(0, 0.02, (64, 256)).astype(np.float16)
    _, _, z2 = O.quantize_asym(W2, 128)
    assert np.array_equal(bits16(z2), f16_bits_nearest(np.round(z2.astype(np.float64))))
    assert np.all((z2.astype(np.float64) >= 0) & (z2.astype(np.float64) <= 15))


def test_constant_groups_golden(golden_dir):
    for variant, c, sbits, z, q, wq in _read_golden(golden_dir, "constant_groups.txt"):
        w = np.full((1, 128), float(c), dtype=np.float16)
        codes, scales, zeros = O.pseudo_quantize(w, 128, zero_point=(variant == "asym"))
        assert int(bits16(scales)[0, 0]) == int(sbits, 16)
        if zeros is not None:
            assert float(zeros[0, 0]) == float(z)
        assert np.all(codes == int(q))
        deq = O.dequant(codes, scales, zeros, 128)
        assert np.all(deq.astype(np.float64) == float(wq))


# ----------------------------------------------------------------------------
# quantize: brute force on small groups
# ----------------------------------------------------------------------------
def _test_groups(rng):
    """fp16 groups [n, 128] over several distributions and degenerate cases."""
    g = []
    g.append(rng.normal(0, 0.02, (64, 128)))
    x = rng.normal(0, 0.02, (32, 128)); x[:, rng.choice(128, 3, replace=False)] *= 10; g.append(x)
    g.append(rng.uniform(0.1, 2.0, (16, 128)))                # all positive: z clamps to 0
    g.append(-rng.uniform(0.1, 2.0, (16, 128)))               # all negative: z clamps to 15
    g.append(rng.uniform(-1e-6, 1e-6, (16, 128)))             # fp16 subnormals
    g.append(rng.uniform(-6e4, 6e4, (8, 128)))                # near the fp16 range
    g.append(np.round(rng.uniform(-8, 8, (16, 128))) / 2)     # many exact ties
    g.append(np.full((4, 128), 0.3))
    return np.concatenate(g).astype(np.float16)


def _argmin_even(err, offsets):
    """Index of the smallest error along the last axis; exact ties go to the
    candidate whose offset is even."""
    best = err.min(axis=-1, keepdims=True)
    cand = (err == best)
    even = cand & (offsets % 2 == 0)
    pick = np.where(even.any(axis=-1, keepdims=True), even, cand)
    return pick.argmax(axis=-1)


def test_asym_codes_are_nearest_level():
    rng = np.random.default_rng(1)
    W = _test_groups(rng)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        codes, scales, zeros = O.quantize_asym(W, 128)
    sf = f16_value(bits16(scales))[0, :]       # one group per row: scales [1, n]
    z = zeros.astype(np.float64)[0, :]
    w = W.astype(np.float64)
    levels = np.arange(16, dtype=np.float64)
    # each code minimizes |(q - z) s - w| over q in 0..15; ties -> even (q - z)
    err = np.abs((levels[None, None, :] - z[:, None, None]) * sf[:, None, None] - w[:, :, None])
    off = levels[None, None, :] - z[:, None, None]
    assert np.array_equal(codes.astype(np.int64), _argmin_even(err, off))
    # the zero point is the level that represents the group minimum
    mn = w.min(axis=1)
    zerr = np.abs(levels[None, :] * sf[:, None] + mn[:, None])
    assert np.array_equal(z.astype(np.int64), _argmin_even(zerr, levels[None, :]))


def test_sym_codes_are_nearest_level():
    rng = np.random.default_rng(2)
    W = _test_groups(rng)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        codes, scales = O.quantize_sym(W, 128)
    sf = f16_value(bits16(scales))[0, :]
    w = W.astype(np.float64)
    c = np.arange(-8, 8, dtype=np.float64)
    err = np.abs(c[None, None, :] * sf[:, None, None] - w[:, :, None])
    assert np.array_equal(codes.astype(np.int64) - 8, _argmin_even(err, c[None, None, :]) - 8)


def _check_scale(s16_bits, r):
    """s16 is the fp16 nearest to r (exact rational), or, when r lies within
    the fp32 rounding window of a half-way point, one of its two neighbours."""
    r = np.asarray(r, dtype=np.float64)
    assert np.all(r > 0)
    near = f16_bits_nearest(r)
    hi = np.clip(np.searchsorted(_VALS, r, side="left"), 1, len(_VALS) - 1)
    lo = hi - 1
    mid = (_VALS[lo] + _VALS[hi]) / 2
    window = np.abs(r - mid) <= r * 2.0 ** -22
    neighbour = (s16_bits == _BITS[lo]) | (s16_bits == _BITS[hi])
    assert np.all((s16_bits == near) | (window & neighbour))


def test_scale_rule_asym_and_sym():
    rng = np.random.default_rng(3)
    W = _test_groups(rng)
    w = W.astype(np.float64)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        _, s_a, _ = O.quantize_asym(W, 128)
        _, s_s = O.quantize_sym(W, 128)
    floor = float(np.float32(1e-5))
    r_a = np.maximum((w.max(1) - w.min(1)) / 15.0, floor)
    r_s = np.maximum(np.abs(w).max(1) / 7.0, floor)
    _check_scale(bits16(s_a)[0, :], r_a)
    _check_scale(bits16(s_s)[0, :], r_s)


def test_dequant_error_bound():
    """|w' - w| <= s/2 + half an fp16 ulp of w' for every element whose level
    was not clipped."""
    rng = np.random.default_rng(4)
    W = _test_groups(rng)[:-1]
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        for zp in (True, False):
            codes, scales, zeros = O.pseudo_quantize(W, 128, zp)
            wq = O.dequant(codes, scales, zeros, 128).astype(np.float64)
            sf = f16_value(bits16(scales)).T.repeat(128, axis=1)      # [n, 128]
            z = (zeros.astype(np.float64).T if zp else np.full(scales.T.shape, 8.0)).repeat(128, axis=1)
            w = W.astype(np.float64)
            lo, hi = (0 - z) * sf, (15 - z) * sf
            inside = (w >= lo - sf / 2) & (w <= hi + sf / 2)
            ulp = np.abs(wq) * 2.0 ** -11 + 2.0 ** -25
            assert np.all(np.abs(wq - w)[inside] <= (sf / 2 + ulp)[inside])


def test_quantize_scale_equivariance():
    """Multiplying a whole group by a power of two multiplies its scale by it
    and keeps codes and zero points (the scale-migration step of the AutoAWQ
    tour, "The big picture", moves such factors between x and W)."""
    rng = np.random.default_rng(5)
    # magnitudes in [2^-6, 4] stay fp16-normal after scaling by 2^-3 .. 2^3
    W = (rng.choice([-1.0, 1.0], (16, 512)) * rng.uniform(2.0 ** -6, 4.0, (16, 512))).astype(np.float16)
    e = rng.integers(-3, 4, size=(16, 4))
    W2 = (W.astype(np.float64) * np.ldexp(1.0, e).repeat(128, axis=1)).astype(np.float16)
    assert np.array_equal(W2.astype(np.float64), W.astype(np.float64) * np.ldexp(1.0, e).repeat(128, axis=1))
    for zp in (True, False):
        c1, s1, z1 = O.pseudo_quantize(W, 128, zp)
        c2, s2, z2 = O.pseudo_quantize(W2, 128, zp)
        assert np.array_equal(c1, c2)
        assert np.array_equal(s2.astype(np.float64), s1.astype(np.float64) * np.ldexp(1.0, e).T)
        if zp:
            assert np.array_equal(z1, z2)


# ----------------------------------------------------------------------------
# pack / unpack ("AWQ > Implementation", "Understanding the Quantization
# Structure": eight 4-bit codes per int32)
# ----------------------------------------------------------------------------
def _slot_of_k(k):
    """Slot of k offset 0..7 in the documented order: even k -> k/2, odd
    k -> 4 + (k-1)/2."""
    return k // 2 if k % 2 == 0 else 4 + (k - 1) // 2


def test_pack_golden_words(golden_dir):
    for r in _read_golden(golden_dir, "pack_words.txt"):
        codes = np.array([[int(c) for c in r[:8]]], dtype=np.uint8)
        word = O.pack(codes)
        assert word.dtype == np.int32
        assert int(word.view(np.uint32)[0, 0]) == int(r[8], 16)
        assert np.array_equal(O.unpack(word), codes)


def test_pack_every_slot_every_value():
    for k in range(8):
        for v in range(16):
            codes = np.zeros((1, 8), dtype=np.uint8)
            codes[0, k] = v
            word = int(O.pack(codes).view(np.uint32)[0, 0])
            assert word == v << (4 * _slot_of_k(k))
            assert np.array_equal(O.unpack(O.pack(codes)), codes)


def test_pack_roundtrip_random():
    rng = np.random.default_rng(6)
    codes = rng.integers(0, 16, size=(37, 1024), dtype=np.uint8)
    assert np.array_equal(O.unpack(O.pack(codes)), codes)
    words = rng.integers(0, 2 ** 32, size=(5, 64), dtype=np.uint64).astype(np.uint32).view(np.int32)
    assert np.array_equal(O.pack(O.unpack(words)), words)


def test_compression_arithmetic():
    """numel*8 weights, fp16 2 bytes each, int32 4 bytes -> 4x ("AWQ >
    Implementation", "Understanding the Quantization Structure")."""
    W, _ = make_layer(512, 512, 1, 0.02)
    qweight, scales, zeros = O.quantize_pack(W, 128, True)
    num_weights = qweight.size * 8
    assert num_weights == W.size
    fp16_size = num_weights * 2
    int4_size = qweight.size * 4
    assert fp16_size / int4_size == 4
    assert qweight.nbytes == int4_size
    assert scales.shape == zeros.shape == (4, 512)        # group-major [K/128, N]


# ----------------------------------------------------------------------------
# matmul and the whole layer
# ----------------------------------------------------------------------------
def test_matmul_exact_integers():
    rng = np.random.default_rng(7)
    x = rng.integers(-4, 5, size=(3, 256)).astype(np.float16)
    w = rng.integers(-8, 9, size=(10, 256)).astype(np.float16)
    y = O.matmul_f64(x, w)
    xi = x.astype(np.int64).tolist()
    wi = w.astype(np.int64).tolist()
    ref = [[sum(a * b for a, b in zip(xr, wr)) for wr in wi] for xr in xi]
    assert y.tolist() == [[float(v) for v in r] for r in ref]


def test_linear_bruteforce_tiny():
    """Whole layer on a tiny case with pure-Python exact arithmetic: nibbles
    read from the words by the documented slot order, decoded with the fp16
    rounding above, summed as fractions."""
    N, K, M = 6, 256, 3
    rng = np.random.default_rng(8)
    for zp in (True, False):
        qweight, scales, zeros = make_packed_random(N, K, 128, zp, seed=9)
        x = rng.standard_normal((M, K)).astype(np.float16)
        y = O.linear(x, qweight, scales, zeros, 128)
        words = qweight.view(np.uint32)
        sv = f16_value(bits16(scales))
        for n in range(N):
            wrow = []
            for k in range(K):
                q = (int(words[n, k // 8]) >> (4 * _slot_of_k(k % 8))) & 0xF
                zz = float(zeros[k // 128, n]) if zp else 8.0
                wrow.append(f16_value(f16_bits_nearest((q - zz) * sv[k // 128, n])))
            for m in range(M):
                exact = sum(Fraction(float(x[m, k])) * Fraction(float(wrow[k])) for k in range(K))
                assert abs(y[m, n] - float(exact)) <= 1e-12 * max(1.0, abs(float(exact)))


def test_scale_migration_invariant():
    """(x / s) (W diag(s))^T == x W^T: exact for power-of-two s, equal within
    float64 rounding otherwise (AutoAWQ tour, "The big picture")."""
    rng = np.random.default_rng(10)
    K = 384
    x = rng.standard_normal((4, K))
    W = rng.standard_normal((K, K))                  # square, so a transposed operand would still run
    s = np.ldexp(1.0, rng.integers(-4, 5, size=K))
    y0 = O.matmul_f64(x, W)
    y1 = O.matmul_f64(x / s, W * s)
    assert np.array_equal(y0, y1)
    s2 = rng.uniform(0.5, 2.0, size=K)
    y2 = O.matmul_f64(x / s2, W * s2)
    assert np.allclose(y2, y0, rtol=1e-12, atol=1e-12 * np.abs(y0).max())
    # the invariant fails for the wrong contraction
    assert not np.allclose(np.asarray(x / s) @ (W * s), np.asarray(x) @ W)


def test_error_metrics():
    y_ref = np.array([[3.0, 4.0]])
    assert O.rel_frobenius(y_ref, y_ref) == 0.0
    assert abs(O.rel_frobenius(np.array([[3.0, 4.05]]), y_ref) - 0.01) < 1e-12
    assert abs(O.max_abs_ratio(np.array([[3.0, 4.05]]), y_ref) - 0.0125) < 1e-12


def test_input_recipe_is_seeded():
    W1, x1 = make_layer(64, 256, 2, 0.02, 0.01, seed=0)
    W2, x2 = make_layer(64, 256, 2, 0.02, 0.01, seed=0)
    assert W1.dtype == np.float16 and x1.dtype == np.float16
    assert np.array_equal(W1.view(np.uint16), W2.view(np.uint16))
    assert np.array_equal(x1.view(np.uint16), x2.view(np.uint16))
    # W does not depend on M
    W3, _ = make_layer(64, 256, 7, 0.02, 0.01, seed=0)
    assert np.array_equal(W1.view(np.uint16), W3.view(np.uint16))
    # salient columns: ceil(1% of K) columns carry about 10x the spread
    Wb = make_weight(2048, 512, 0.02, 0.01, seed=0).astype(np.float64)
    col = Wb.std(axis=0)
    assert (col > 0.1).sum() == 6 and (col < 0.03).sum() == 512 - 6
