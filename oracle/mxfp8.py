"""MXFP8 codec and block quantiser, fp64 (oracle; test infrastructure only).

What the pages fix: MXFP8 keeps 8 bits per value and gives every block of 32 values
its own scale factor ("MoE-Training für biologische Grundmodelle optimieren",
hyper.ai/de, passage on MXFP8; "NVIDIA optimise l'entraînement MoE des modèles
biologiques", hyper.ai/fr, passage on MXFP8 halving the footprint). Everything else
is a reading, stated where it is used:

* element format: OCP FP8 E4M3 (bias 7, 3 mantissa bits, subnormals, max 448, no
  infinities, S.1111.111 is NaN);
* scale: an E8M0 power of two, exponent X = clamp(floor(log2(amax)) - 8, -127, 127)
  (8 = largest exponent of E4M3), stored as the byte X + 127; amax == 0 -> byte 0;
* element: E4M3(v * 2^-X), round to nearest, ties to even, saturating to +-448;
  the sign is kept, so a negative value that rounds to zero is 0x80;
* block direction: 32 consecutive values along the contraction dimension of the
  GEMM that consumes the tensor ("rowwise" = along columns; "colwise" = 32 rows of
  one expert segment, stored transposed).

The E5M2 element format is the variant for gradients (the pages name FP8 beside MXFP8
and fix neither element format; OCP FP8 E5M2: bias 15, 2 mantissa bits, subnormals,
max 57344, S.11111.00 infinite, S.11111.xx with xx != 0 NaN). Its scale rule is the same
with the format's largest exponent: X = clamp(floor(log2(amax)) - 15, -127, 127); its
elements saturate to +-57344.

The "ceil" scale rule is a variant of the scale choice (the pages give none): the
smallest power of two for which no element of the block exceeds the format's largest
value, so nothing saturates (the OCP exponent, plus one when the block's amax lies
above that value times the OCP scale).

The encoder is a nearest-value search over the table of finite codes; it never uses
bit manipulation, so that it is independent of the decoder's closed form.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8          # floor(log2(448))
E5M2_MAX = 57344.0
E5M2_EMAX = 15         # floor(log2(57344))
SCALE_BIAS = 127
SCALE_MIN_EXP = -127
SCALE_MAX_EXP = 127
BLOCK = 32


def e4m3_decode(code):
    """Closed form of OCP E4M3: (-1)^s * 2^(e-7) * (1 + m/8), subnormal 2^-6 * m/8."""
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


# Non-negative finite codes 0x00..0x7E and their values, ascending (the decoder is
# monotone on them, which the tests check).
_POS_CODES = np.arange(0x7F, dtype=np.int64)
_POS_VALUES = e4m3_decode(_POS_CODES)


def _nearest_code(x, pos_codes, pos_values, vmax):
    """Nearest code of a table of non-negative finite values (ascending) to each fp64
    value; ties go to the even code (mantissa LSB 0); magnitudes beyond vmax saturate to
    the largest code; the sign bit (0x80) follows the input's sign."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("fp8 encode: non-finite input")
    a = np.abs(x)
    hi = np.searchsorted(pos_values, a, side="left")        # first value >= a
    hi = np.minimum(hi, len(pos_values) - 1)
    lo = np.maximum(hi - 1, 0)
    vlo, vhi = pos_values[lo], pos_values[hi]
    dlo, dhi = a - vlo, vhi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((pos_codes[hi] & 1) == 0))
    code = np.where(pick_hi, pos_codes[hi], pos_codes[lo])
    code = np.where(a >= vhi, pos_codes[hi], code)           # exact hit / above table top
    code = np.where(a >= vmax, pos_codes[-1], code)          # saturate
    neg = np.signbit(x)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def e4m3_encode(x):
    """Nearest E4M3 code to each fp64 value; ties go to the even code (mantissa LSB 0);
    magnitudes beyond 448 saturate to 448; the sign bit follows the input's sign."""
    return _nearest_code(x, _POS_CODES, _POS_VALUES, E4M3_MAX)


def e5m2_decode(code):
    """Closed form of OCP E5M2: (-1)^s * 2^(e-15) * (1 + m/4), subnormal 2^-14 * m/4;
    exponent field 31 is infinity (m == 0) or NaN."""
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 2) & 0x1F
    m = c & 0x3
    mag = np.where(e == 0, (m / 4.0) * 2.0 ** -14, (1.0 + m / 4.0) * np.exp2(e.astype(np.float64) - 15.0))
    mag = np.where(e == 31, np.where(m == 0, np.inf, np.nan), mag)
    return np.where(s == 1, -mag, mag)


# Non-negative finite E5M2 codes 0x00..0x7B and their values, ascending.
_POS_CODES_E5M2 = np.arange(0x7C, dtype=np.int64)
_POS_VALUES_E5M2 = e5m2_decode(_POS_CODES_E5M2)


def e5m2_encode(x):
    """Nearest E5M2 code to each fp64 value; ties to the even code; magnitudes beyond
    57344 saturate to 57344 (never infinity); the sign bit follows the input's sign."""
    return _nearest_code(x, _POS_CODES_E5M2, _POS_VALUES_E5M2, E5M2_MAX)


# element formats: name -> (encode, decode, largest exponent, largest finite value)
FORMATS = {"e4m3": (e4m3_encode, e4m3_decode, E4M3_EMAX, E4M3_MAX),
           "e5m2": (e5m2_encode, e5m2_decode, E5M2_EMAX, E5M2_MAX)}


def scale_exponent(amax, emax=E4M3_EMAX, rule="ocp", vmax=None):
    """Scale exponent of a block with largest magnitude amax (amax == 0 -> -127, byte 0x00).
    rule "ocp": X = clamp(floor(log2(amax)) - emax, -127, 127), emax = the element
      format's largest exponent (8 for E4M3, 15 for E5M2); elements above vmax * 2^X
      saturate.
    rule "ceil": the smallest X with amax <= vmax * 2^X (vmax = the format's largest
      finite value), clamped likewise: the power-of-two scale rounded up so that no
      element saturates. It is the "ocp" exponent, or one more when amax lies above
      vmax * 2^X_ocp."""
    amax = np.asarray(amax, dtype=np.float64)
    mant, ex = np.frexp(amax)            # amax = mant * 2^ex, mant in [0.5, 1)
    fl = ex.astype(np.int64) - 1         # floor(log2(amax)) for amax > 0
    X = fl - emax
    if rule == "ceil":
        X = X + (amax > vmax * np.exp2(X.astype(np.float64))).astype(np.int64)
    elif rule != "ocp":
        raise ValueError(f"unknown scale rule {rule!r}")
    X = np.clip(X, SCALE_MIN_EXP, SCALE_MAX_EXP)
    return np.where(amax == 0, SCALE_MIN_EXP, X).astype(np.int64)


def quantize_blocks(v, fmt="e4m3", rule="ocp"):
    """Quantise ``v[..., 32]`` block by block -> (codes uint8[..., 32], scale bytes uint8[...])."""
    encode, _, emax, vmax = FORMATS[fmt]
    v = np.asarray(v, dtype=np.float64)
    assert v.shape[-1] == BLOCK
    amax = np.max(np.abs(v), axis=-1)
    X = scale_exponent(amax, emax, rule, vmax)
    scaled = v * np.exp2(-X.astype(np.float64))[..., None]   # exact power-of-two scaling in fp64
    codes = encode(scaled)
    return codes, (X + SCALE_BIAS).astype(np.uint8)


def dequantize_blocks(codes, scale_bytes, fmt="e4m3"):
    """decode(code) * 2^(scale byte - 127), exact in fp64."""
    decode = FORMATS[fmt][1]
    X = scale_bytes.astype(np.int64) - SCALE_BIAS
    return decode(codes) * np.exp2(X.astype(np.float64))[..., None]


def quantize_rowwise(a, fmt="e4m3", rule="ocp"):
    """Blocks of 32 along the last axis of a 2-D matrix [R, C] (C % 32 == 0).
    Returns (codes uint8[R, C], scales uint8[R, C/32])."""
    a = np.asarray(a, dtype=np.float64)
    R, C = a.shape
    assert C % BLOCK == 0
    codes, sc = quantize_blocks(a.reshape(R, C // BLOCK, BLOCK), fmt, rule)
    return codes.reshape(R, C), sc


def dequantize_rowwise(codes, scales, fmt="e4m3"):
    R, C = codes.shape
    return dequantize_blocks(codes.reshape(R, C // BLOCK, BLOCK), scales, fmt).reshape(R, C)


def quantize_colwise_t(a, fmt="e4m3", rule="ocp"):
    """Blocks of 32 consecutive rows in each column of [R, C] (R % 32 == 0), stored
    transposed: (codes uint8[C, R], scales uint8[C, R/32]). The caller lays segments
    out so that no block crosses an expert boundary."""
    a = np.asarray(a, dtype=np.float64)
    return quantize_rowwise(a.T, fmt, rule)


def fake_quant_rowwise(a, fmt="e4m3", rule="ocp"):
    """Quantise then dequantise along rows (used where the oracle needs the value a
    quantised operand stands for)."""
    c, s = quantize_rowwise(a, fmt, rule)
    return dequantize_rowwise(c, s, fmt)


def fake_quant_colwise(a, fmt="e4m3", rule="ocp"):
    """Colwise quantise/dequantise, returned in the original [R, C] orientation."""
    c, s = quantize_colwise_t(a, fmt, rule)
    return dequantize_rowwise(c, s, fmt).T


# ----------------------------------------------------------------------------- per-tensor FP8
# The pages name FP8 beside MXFP8 ("MoE-Training für biologische Grundmodelle optimieren",
# hyper.ai/de, precision passage) without fixing its scaling. Reading: one fp32 scale per
# tensor (per expert for the expert weights), E4M3 elements. The scale is kept as the fp32
# multiplier that maps the tensor's largest magnitude onto E4M3's largest value:
#   m = fp32(448 / amax), rounded to nearest (m = 1 when amax == 0);
#   code = E4M3(fp32(v * m)): the product is rounded to fp32 first, then to E4M3 (nearest,
#   ties to even, saturating to +-448);
#   value = decode(code) / m.
# Rounding the product to fp32 before the E4M3 rounding makes the code a function of two
# fp32 roundings that any fp32 implementation reproduces exactly.

FP32_MAX = float(np.finfo(np.float32).max)


def tensor_multiplier(amax):
    """fp32 multiplier m = 448 / amax rounded to nearest fp32; 1 when amax == 0, and the
    largest finite fp32 when the quotient overflows (amax below about 1.3e-36)."""
    a = np.float32(amax)
    if a == 0:
        return np.float32(1.0)
    with np.errstate(over="ignore"):
        m = np.float32(np.float32(E4M3_MAX) / a)
    return np.float32(min(float(m), FP32_MAX))


def quantize_tensor(v, m):
    """Per-tensor E4M3 codes of fp32-representable values v under the multiplier m."""
    prod = np.asarray(v, dtype=np.float32) * np.float32(m)     # fp32 product, rounded to nearest
    return e4m3_encode(prod.astype(np.float64))


def dequantize_tensor(codes, m):
    """decode(code) / m in fp64."""
    return e4m3_decode(codes) / np.float64(m)


def fake_quant_tensor(v, m):
    return dequantize_tensor(quantize_tensor(v, m), m)
