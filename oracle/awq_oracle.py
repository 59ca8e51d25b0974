"""CPU oracle for the group-wise INT4 weight-only linear layer (W4A16, AWQ style).

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
statement of what the CUDA library computes. Only the test suite, the smoke
check in ``__graft_entry__`` and the CPU-baseline / reference arm of
``bench.py`` may import it. The CUDA product path never imports, links or
calls it, and it shares no code, table or constant generator with the CUDA
sources: the nibble order below is restated here from the documented
format, not imported.

Sources (cited by page title and section):

* "AutoAWQ" code tour (pyshine.com), section "The Quantization Flow Up
  Close": pseudo-quantization rounds each group of weights to integer
  levels against a per-group scale and zero point; section "From Install to
  Your First Model": ``zero_point`` selects asymmetric vs symmetric,
  ``q_group_size`` = 128 weights share one scale (and zero), ``w_bit`` = 4.
* "AWQ > Implementation" (Language AI Handbook), section "Understanding the
  Quantization Structure": ``qweight`` holds eight 4-bit codes per int32,
  scales are fp16, one scale and zero per group of 128 weights.
* "AWQ Quantization Support" (fak explainer), section "Dequantization
  Formula": weight = scale x (code - 8) for the symmetric variant, codes
  0..15.
* "AutoAWQ" code tour, section "The big picture": dividing an input channel
  of x by a constant and multiplying the matching weight column by it leaves
  the layer output unchanged (used as a pin on the matmul, not here).

Readings where the pages are silent:

* Asymmetric scale/zero follow the plain per-group min/max affine rule on
  the levels 0..15; the range is not widened to include 0.
* Quantize arithmetic is IEEE fp32 with round-to-nearest-even, and the
  fp16-rounded scale is the one used to derive the zero point and the codes.
* The fp32 scale is floored at 1e-5 before the fp16 cast (constant groups).
* ``rint`` (ties to even) for every rounding to an integer.
* Symmetric scale = max|w| / 7 (largest positive level 7); codes are
  clamp(rint(w/s), -8, 7) + 8.
* Zero points are stored as fp16 values holding the integers 0..15.
* Scales and zero points are stored group-major, [K/g, N] (entry [j, n] is
  the group of k in [128j, 128j + 128) of output channel n), the orientation
  AutoAWQ's checkpoints use for ``scales``.
* Packing is along K, eight consecutive k per int32 word; nibble slot i
  (bits 4i..4i+3) of the word covering k = 8w..8w+7 holds k = 8w + SLOT_K[i]
  with SLOT_K = (0, 2, 4, 6, 1, 3, 5, 7).

Every function below works on NumPy arrays. fp16 tensors are numpy.float16,
packed words are numpy.int32 (the uint32 bit pattern reinterpreted).
"""

from __future__ import annotations

import numpy as np

GROUP_SIZE = 128
W_BIT = 4
LEVELS = 2 ** W_BIT - 1            # highest code, 15
SYM_ZERO = 8                       # fixed zero point of the symmetric variant
SCALE_FLOOR = np.float32(1e-5)     # reading: floor on the fp32 scale
# Nibble slot i of a packed word holds k offset SLOT_K[i] (documented format).
SLOT_K = (0, 2, 4, 6, 1, 3, 5, 7)


def _groups_f32(W: np.ndarray, group_size: int) -> np.ndarray:
    """View fp16 W[N, K] as fp32 [N, K/g, g] (exact widening)."""
    W = np.asarray(W)
    if W.dtype != np.float16:
        raise TypeError("W must be float16")
    N, K = W.shape
    if group_size <= 0 or K % group_size:
        raise ValueError("K must be a positive multiple of the group size")
    return W.astype(np.float32).reshape(N, K // group_size, group_size)


def quantize_asym(W: np.ndarray, group_size: int = GROUP_SIZE):
    """Asymmetric (zero-point) group quantization of fp16 W[N, K].

    Follows the AutoAWQ tour, "The Quantization Flow Up Close" (round each
    group to integer levels against its scale and zero point) with the
    min/max reading. Per row n and group j, with w the group's values in
    fp32:

      1. mx = max(w), mn = min(w)
      2. s32 = max((mx - mn) / 15, 1e-5)            fp32, round to nearest even
      3. s = fp16(s32); sf = float(s)
      4. z = clamp(-rint(mn / sf), 0, 15)
      5. q = clamp(rint(w / sf) + z, 0, 15)

    Returns (codes uint8 [N, K], scales fp16 [G, N], zeros fp16 [G, N]).
    """
    w = _groups_f32(W, group_size)
    mx = w.max(axis=2)
    mn = w.min(axis=2)
    s32 = np.maximum((mx - mn) / np.float32(LEVELS), SCALE_FLOOR)
    scales = s32.astype(np.float16)
    sf = scales.astype(np.float32)
    z = np.clip(-np.rint(mn / sf), 0, LEVELS).astype(np.float32)
    q = np.clip(np.rint(w / sf[..., None]) + z[..., None], 0, LEVELS)
    codes = q.astype(np.uint8).reshape(W.shape)
    # z is an integer level; storing it through an integer keeps 0 as +0
    # (-rint of a non-negative minimum is -0.0 in floating point).
    zeros = z.astype(np.int32).astype(np.float16)
    return codes, np.ascontiguousarray(scales.T), np.ascontiguousarray(zeros.T)


def quantize_sym(W: np.ndarray, group_size: int = GROUP_SIZE):
    """Symmetric group quantization, zero point fixed at 8.

    The fak explainer, "Dequantization Formula", fixes the decode as
    scale x (code - 8) with codes 0..15; the scale rule is the reading
    s = max|w| / 7. Per row n and group j:

      1. a = max|w|
      2. s32 = max(a / 7, 1e-5); s = fp16(s32); sf = float(s)
      3. c = clamp(rint(w / sf), -8, 7); q = c + 8

    With this scale |w / sf| stays below 7.5 (the fp16 rounding of the scale
    is far smaller than the margin, and the 1e-5 floor only lowers the
    ratio), so code 0 (c = -8) is never produced: 15 of the 16 levels are
    used, as the max/7 reading implies.

    Returns (codes uint8 [N, K], scales fp16 [G, N]).
    """
    w = _groups_f32(W, group_size)
    a = np.abs(w).max(axis=2)
    s32 = np.maximum(a / np.float32(7.0), SCALE_FLOOR)
    scales = s32.astype(np.float16)
    sf = scales.astype(np.float32)
    c = np.clip(np.rint(w / sf[..., None]), -8, 7)
    codes = (c + SYM_ZERO).astype(np.uint8).reshape(W.shape)
    return codes, np.ascontiguousarray(scales.T)


def pseudo_quantize(W: np.ndarray, group_size: int = GROUP_SIZE, zero_point: bool = True):
    """Quantize with the variant ``zero_point`` selects (AutoAWQ tour, "From
    Install to Your First Model"). Returns (codes, scales, zeros-or-None)."""
    if zero_point:
        return quantize_asym(W, group_size)
    codes, scales = quantize_sym(W, group_size)
    return codes, scales, None


def pack(codes: np.ndarray) -> np.ndarray:
    """Pack 4-bit codes [N, K] into int32 words [N, K/8], eight per word
    ("AWQ > Implementation", "Understanding the Quantization Structure").

    Word w of a row covers k = 8w .. 8w+7; nibble slot i holds k = 8w +
    SLOT_K[i].
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    if K % 8:
        raise ValueError("K must be a multiple of 8")
    if codes.size and (codes.min() < 0 or codes.max() > LEVELS):
        raise ValueError("codes must lie in 0..15")
    c = codes.astype(np.uint32).reshape(N, K // 8, 8)
    word = np.zeros((N, K // 8), dtype=np.uint32)
    for slot, koff in enumerate(SLOT_K):
        word |= c[:, :, koff] << np.uint32(4 * slot)
    return word.view(np.int32)


def unpack(qweight: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack`: int32 words [N, K/8] -> uint8 codes [N, K]."""
    qweight = np.asarray(qweight)
    if qweight.dtype != np.int32:
        raise TypeError("qweight must be int32")
    N, W = qweight.shape
    word = qweight.view(np.uint32)
    codes = np.zeros((N, W, 8), dtype=np.uint8)
    for slot, koff in enumerate(SLOT_K):
        codes[:, :, koff] = (word >> np.uint32(4 * slot)) & np.uint32(0xF)
    return codes.reshape(N, W * 8)


def dequant(codes: np.ndarray, scales: np.ndarray, zeros, group_size: int = GROUP_SIZE) -> np.ndarray:
    """fp16 weights w' = fp16((q - z) * s); z = 8 when ``zeros`` is None.
    ``scales`` and ``zeros`` are [G, N].

    Asymmetric: (q - z[n, j]) * s[n, j] (the zero-point decode the AutoAWQ
    tour names); symmetric: scale x (code - 8) (fak explainer,
    "Dequantization Formula"). (q - z) * s is exact in fp32 (|q - z| <= 15
    times an 11-bit significand), so the only rounding is the one cast to
    fp16, round to nearest even.
    """
    codes = np.asarray(codes)
    N, K = codes.shape
    G = K // group_size
    q = codes.astype(np.float32).reshape(N, G, group_size)
    sf = np.asarray(scales).astype(np.float32).reshape(G, N).T.reshape(N, G, 1)
    if zeros is None:
        z = np.float32(SYM_ZERO)
    else:
        z = np.asarray(zeros).astype(np.float32).reshape(G, N).T.reshape(N, G, 1)
    return ((q - z) * sf).astype(np.float16).reshape(N, K)


def matmul_f64(x: np.ndarray, Wd: np.ndarray) -> np.ndarray:
    """y[m, n] = sum_k x[m, k] * w'[n, k], the plain definition in float64."""
    return np.asarray(x).astype(np.float64) @ np.asarray(Wd).astype(np.float64).T


def linear(x: np.ndarray, qweight: np.ndarray, scales: np.ndarray, zeros,
           group_size: int = GROUP_SIZE) -> np.ndarray:
    """The W4A16 linear layer: unpack, dequantize, then the float64 matmul."""
    return matmul_f64(x, dequant(unpack(qweight), scales, zeros, group_size))


def quantize_pack(W: np.ndarray, group_size: int = GROUP_SIZE, zero_point: bool = True):
    """Quantize then pack: (qweight int32 [N, K/8], scales, zeros-or-None)."""
    codes, scales, zeros = pseudo_quantize(W, group_size, zero_point)
    return pack(codes), scales, zeros


def rel_frobenius(y: np.ndarray, y_ref: np.ndarray) -> float:
    """||y - y_ref||_F / ||y_ref||_F in float64."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    den = np.linalg.norm(y_ref)
    return float(np.linalg.norm(y - y_ref) / den) if den > 0 else float(np.linalg.norm(y))


def max_abs_ratio(y: np.ndarray, y_ref: np.ndarray) -> float:
    """max|y - y_ref| / max|y_ref| in float64."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    den = np.abs(y_ref).max() if y_ref.size else 0.0
    num = np.abs(y - y_ref).max() if y_ref.size else 0.0
    return float(num / den) if den > 0 else float(num)


# ---------------------------------------------------------------------------
# Fused MLP input projection ("AutoAWQ" code tour, "The Quantization Flow Up
# Close": the fuser merges the gate and up projections into one quantized MLP
# block; "AutoAWQ" capability page: fused blocks cut launches and
# intermediate tensors). Reading: the activation is SiLU, that of the
# Llama-family MLP whose fuser the tour names; h = silu(gate) * up.
# ---------------------------------------------------------------------------
TILE_ROWS = 16   # rows per tile of the interleaved gate/up layout (documented format)


def silu_f64(v: np.ndarray) -> np.ndarray:
    """SiLU in float64: v * sigmoid(v) = v / (1 + exp(-v))."""
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore"):
        return v / (1.0 + np.exp(-v))


def gate_up_silu_f64(x: np.ndarray, Wg_d: np.ndarray, Wu_d: np.ndarray) -> np.ndarray:
    """h[m, n] = silu(sum_k x[m,k] w'g[n,k]) * sum_k x[m,k] w'u[n,k], both
    products by the plain float64 definition."""
    return silu_f64(matmul_f64(x, Wg_d)) * matmul_f64(x, Wu_d)


def interleave_gate_up(a_gate: np.ndarray, a_up: np.ndarray, axis: int = 0) -> np.ndarray:
    """The fused weight layout: along ``axis`` (rows of qweight, columns of the
    group-major scales and zeros), 16-row tiles alternate gate, up: tile 2j
    holds gate rows 16j .. 16j+15, tile 2j+1 holds up rows 16j .. 16j+15.
    Needs the row count to be a multiple of 16."""
    a_gate = np.moveaxis(np.asarray(a_gate), axis, 0)
    a_up = np.moveaxis(np.asarray(a_up), axis, 0)
    n = a_gate.shape[0]
    if a_up.shape != a_gate.shape or n % TILE_ROWS:
        raise ValueError("gate and up need the same shape and a multiple of 16 rows")
    out = np.empty((2 * n,) + a_gate.shape[1:], dtype=a_gate.dtype)
    for j in range(n // TILE_ROWS):
        out[2 * j * TILE_ROWS:(2 * j + 1) * TILE_ROWS] = a_gate[j * TILE_ROWS:(j + 1) * TILE_ROWS]
        out[(2 * j + 1) * TILE_ROWS:(2 * j + 2) * TILE_ROWS] = a_up[j * TILE_ROWS:(j + 1) * TILE_ROWS]
    return np.moveaxis(out, 0, axis)


# ---------------------------------------------------------------------------
# Activation-aware scale search ("AutoAWQ" code tour, "The Quantization Flow
# Up Close": the search computes a per-channel mean of normalized weights and
# a float32 mean of activations, runs the fp16 module once as the reference,
# and picks the candidate scaling with the lowest output error; "From Install
# to Your First Model": duo_scaling uses both the weight and the activation
# statistics; "The big picture": dividing an input channel of x by s and
# multiplying the matching weight column by s leaves the output unchanged).
#
# Readings (the pages give no formula or grid):
# * candidates s(alpha) = mean|x|^alpha / (mean|w^|^(1 - alpha) + 1e-4) with
#   duo scaling, mean|x|^alpha without, for alpha = i / n_grid, i = 0 ..
#   n_grid - 1; each floored at 1e-4 and divided by sqrt(max(s) * min(s)) so
#   the scaled weights stay in fp16 range;
# * w^ = |w| / (max |w| over its group of 128 in the same row), 0 for an
#   all-zero group; mean|w^| is over the N rows;
# * all of the statistics and candidate arithmetic in fp32;
# * error = mean over outputs of (y_ref - y)^2, y_ref = fp16(x . W^T) (the
#   fp16 module), y = fp16((x / s) . Q(W diag(s))'^T), x / s and W diag(s)
#   rounded to fp16;
# * the first minimum wins a tie.
# ---------------------------------------------------------------------------
SCALE_EPS = np.float32(1e-4)


def act_mean_abs(X: np.ndarray) -> np.ndarray:
    """mean over rows of |x[m, k]|, fp32 [K]."""
    return np.abs(np.asarray(X).astype(np.float32)).mean(axis=0, dtype=np.float32)


def weight_norm_mean(W: np.ndarray, group_size: int = GROUP_SIZE) -> np.ndarray:
    """mean over rows n of |w[n, k]| / max|w[n, group of k]|, fp32 [K]."""
    A = np.abs(_groups_f32(W, group_size))                    # [N, G, g]
    mx = A.max(axis=2, keepdims=True)
    Wn = np.divide(A, mx, out=np.zeros_like(A), where=mx > 0)
    N, G, g = Wn.shape
    return Wn.reshape(N, G * g).mean(axis=0, dtype=np.float32)


def candidate_scales(x_mean: np.ndarray, w_mean: np.ndarray, alpha: float, duo: bool = True) -> np.ndarray:
    """The scale vector of one grid point, fp32 [K]."""
    a = np.float32(alpha)
    s = np.power(x_mean.astype(np.float32), a)
    if duo:
        s = s / (np.power(w_mean.astype(np.float32), np.float32(1.0) - a) + SCALE_EPS)
    s = np.maximum(s.astype(np.float32), SCALE_EPS)
    return (s / np.sqrt(s.max() * s.min())).astype(np.float32)


def scaled_output(W: np.ndarray, X: np.ndarray, s: np.ndarray, group_size: int = GROUP_SIZE,
                  zero_point: bool = True) -> np.ndarray:
    """fp16((x / s) . Q(W diag(s))'^T): the quantized module with the scale
    folded into its weights and divided out of its input."""
    s = s.astype(np.float32)
    Ws = (np.asarray(W).astype(np.float32) * s[None, :]).astype(np.float16)
    Xs = (np.asarray(X).astype(np.float32) / s[None, :]).astype(np.float16)
    codes, sc, z = pseudo_quantize(Ws, group_size, zero_point)
    return matmul_f64(Xs, dequant(codes, sc, z, group_size)).astype(np.float16)


def search_scale(W: np.ndarray, X: np.ndarray, group_size: int = GROUP_SIZE, zero_point: bool = True,
                 n_grid: int = 20, duo: bool = True):
    """(best scales fp32 [K], losses [n_grid] float64, best index)."""
    y_ref = matmul_f64(X, W).astype(np.float16).astype(np.float64)
    x_mean, w_mean = act_mean_abs(X), weight_norm_mean(W, group_size)
    losses = np.empty(n_grid)
    for i in range(n_grid):
        s = candidate_scales(x_mean, w_mean, i / n_grid, duo)
        y = scaled_output(W, X, s, group_size, zero_point).astype(np.float64)
        losses[i] = np.mean((y_ref - y) ** 2)
    best = int(np.argmin(losses))
    return candidate_scales(x_mean, w_mean, best / n_grid, duo), losses, best


# ---------------------------------------------------------------------------
# Clip search ("AutoAWQ" code tour, "The Quantization Flow Up Close": the
# clipping pass shrinks extreme values group by group where that lowers the
# output error; apply_clip switches it). Readings (the pages give no grid or
# criterion formula):
# * ratio grid r_i = 1 - max_shrink * i / n_grid, i = 0 .. n_grid - 1;
# * a group of row n is clipped to [-t, t], t = r * max|w| of the group (fp32),
#   and the clipped values rounded to fp16, then quantized as usual;
# * error of (row n, group j) = sum over calibration rows m of
#   (x[m, group j] . (w - w'))^2 = d^T (X_j^T X_j) d, d = w - w' in float64;
# * per (row, group) the first ratio with the lowest error wins.
# ---------------------------------------------------------------------------
def clip_groups(W: np.ndarray, ratios: np.ndarray, group_size: int = GROUP_SIZE) -> np.ndarray:
    """fp16 W clipped per (row, group) to [-t, t], t = ratio * max|w| of the
    group; ratios [G, N] (group-major, as the scales)."""
    A = _groups_f32(W, group_size)                                   # [N, G, g]
    t = np.abs(A).max(axis=2) * np.asarray(ratios, np.float32).T     # [N, G] fp32
    C = np.clip(A, -t[:, :, None], t[:, :, None]).astype(np.float16)
    return C.reshape(np.asarray(W).shape)


def search_clip(W: np.ndarray, X: np.ndarray, group_size: int = GROUP_SIZE, zero_point: bool = True,
                n_grid: int = 20, max_shrink: float = 0.5):
    """(best ratios fp32 [G, N], errors float64 [n_grid, G, N])."""
    N, K = np.asarray(W).shape
    G = K // group_size
    Xg = np.asarray(X).astype(np.float64).reshape(-1, G, group_size)
    gram = np.einsum("mja,mjb->jab", Xg, Xg)                         # [G, g, g]
    Wf = np.asarray(W).astype(np.float64).reshape(N, G, group_size)
    errs = np.empty((n_grid, G, N))
    for i in range(n_grid):
        r = np.float32(1.0) - np.float32(max_shrink) * np.float32(i) / np.float32(n_grid)
        Wc = clip_groups(W, np.full((G, N), r, np.float32), group_size)
        codes, sc, z = pseudo_quantize(Wc, group_size, zero_point)
        D = Wf - dequant(codes, sc, z, group_size).astype(np.float64).reshape(N, G, group_size)
        errs[i] = np.einsum("nja,jab,njb->jn", D, gram, D)
    best = np.argmin(errs, axis=0)                                    # first minimum
    ratios = (np.float32(1.0) - np.float32(max_shrink) * best.astype(np.float32) / np.float32(n_grid))
    return ratios.astype(np.float32), errs


# ---------------------------------------------------------------------------
# Packed zero points ("AWQ > Implementation", "Understanding the Quantization
# Structure": a quantized layer holds ``qweight``, ``scales`` and ``qzeros``;
# its 4-bit values are stored eight per int32).
#
# Readings (the pages name ``qzeros`` but give neither its axis nor its nibble
# order):
# * qzeros is group-major like the scales, [G, N/8]: word w of group row j
#   covers output channels n = 8w .. 8w+7, and nibble i (bits 4i..4i+3) holds
#   n = 8w + i (the plain order: unlike the codes, no decode trick depends on
#   it);
# * a zero point that is not an integer in 0..15 is rounded to the nearest
#   integer (ties to even) and clamped to 0..15; NaN becomes 0.
# ---------------------------------------------------------------------------
def pack_zeros(zeros: np.ndarray) -> np.ndarray:
    """fp16 zero points [G, N] -> int32 qzeros [G, N/8] (N % 8 == 0)."""
    z = np.asarray(zeros).astype(np.float32)
    G, N = z.shape
    if N % 8:
        raise ValueError("N must be a multiple of 8")
    z = np.where(np.isnan(z), np.float32(0.0), z)
    q = np.clip(np.rint(z), 0, LEVELS).astype(np.uint32).reshape(G, N // 8, 8)
    word = np.zeros((G, N // 8), dtype=np.uint32)
    for i in range(8):
        word |= q[:, :, i] << np.uint32(4 * i)
    return word.view(np.int32)


def unpack_zeros(qzeros: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_zeros`: int32 [G, N/8] -> fp16 zero points [G, N]."""
    qzeros = np.asarray(qzeros)
    if qzeros.dtype != np.int32:
        raise TypeError("qzeros must be int32")
    G, W = qzeros.shape
    word = qzeros.view(np.uint32)
    out = np.zeros((G, W, 8), dtype=np.float16)
    for i in range(8):
        out[:, :, i] = ((word >> np.uint32(4 * i)) & np.uint32(0xF)).astype(np.float16)
    return out.reshape(G, W * 8)
