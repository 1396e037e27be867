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

The encoder is a nearest-value search over the table of finite codes; it never uses
bit manipulation, so that it is independent of the decoder's closed form.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_EMAX = 8          # floor(log2(448))
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


def e4m3_encode(x):
    """Nearest E4M3 code to each fp64 value; ties go to the even code (mantissa LSB 0);
    magnitudes beyond 448 saturate to 448; the sign bit follows the input's sign."""
    x = np.asarray(x, dtype=np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode: non-finite input")
    a = np.abs(x)
    hi = np.searchsorted(_POS_VALUES, a, side="left")       # first value >= a
    hi = np.minimum(hi, len(_POS_VALUES) - 1)
    lo = np.maximum(hi - 1, 0)
    vlo, vhi = _POS_VALUES[lo], _POS_VALUES[hi]
    dlo, dhi = a - vlo, vhi - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & ((_POS_CODES[hi] & 1) == 0))
    code = np.where(pick_hi, _POS_CODES[hi], _POS_CODES[lo])
    code = np.where(a >= vhi, _POS_CODES[hi], code)          # exact hit / above table top
    code = np.where(a >= E4M3_MAX, 0x7E, code)               # saturate
    neg = np.signbit(x)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def scale_exponent(amax):
    """X = clamp(floor(log2(amax)) - 8, -127, 127); amax == 0 -> -127 (byte 0x00)."""
    amax = np.asarray(amax, dtype=np.float64)
    mant, ex = np.frexp(amax)            # amax = mant * 2^ex, mant in [0.5, 1)
    fl = ex.astype(np.int64) - 1         # floor(log2(amax)) for amax > 0
    X = np.clip(fl - E4M3_EMAX, SCALE_MIN_EXP, SCALE_MAX_EXP)
    return np.where(amax == 0, SCALE_MIN_EXP, X).astype(np.int64)


def quantize_blocks(v):
    """Quantise ``v[..., 32]`` block by block -> (codes uint8[..., 32], scale bytes uint8[...])."""
    v = np.asarray(v, dtype=np.float64)
    assert v.shape[-1] == BLOCK
    amax = np.max(np.abs(v), axis=-1)
    X = scale_exponent(amax)
    scaled = v * np.exp2(-X.astype(np.float64))[..., None]   # exact power-of-two scaling in fp64
    codes = e4m3_encode(scaled)
    return codes, (X + SCALE_BIAS).astype(np.uint8)


def dequantize_blocks(codes, scale_bytes):
    """decode(code) * 2^(scale byte - 127), exact in fp64."""
    X = scale_bytes.astype(np.int64) - SCALE_BIAS
    return e4m3_decode(codes) * np.exp2(X.astype(np.float64))[..., None]


def quantize_rowwise(a):
    """Blocks of 32 along the last axis of a 2-D matrix [R, C] (C % 32 == 0).
    Returns (codes uint8[R, C], scales uint8[R, C/32])."""
    a = np.asarray(a, dtype=np.float64)
    R, C = a.shape
    assert C % BLOCK == 0
    codes, sc = quantize_blocks(a.reshape(R, C // BLOCK, BLOCK))
    return codes.reshape(R, C), sc


def dequantize_rowwise(codes, scales):
    R, C = codes.shape
    return dequantize_blocks(codes.reshape(R, C // BLOCK, BLOCK), scales).reshape(R, C)


def quantize_colwise_t(a):
    """Blocks of 32 consecutive rows in each column of [R, C] (R % 32 == 0), stored
    transposed: (codes uint8[C, R], scales uint8[C, R/32]). The caller lays segments
    out so that no block crosses an expert boundary."""
    a = np.asarray(a, dtype=np.float64)
    return quantize_rowwise(a.T)


def fake_quant_rowwise(a):
    """Quantise then dequantise along rows (used where the oracle needs the value a
    quantised operand stands for)."""
    c, s = quantize_rowwise(a)
    return dequantize_rowwise(c, s)


def fake_quant_colwise(a):
    """Colwise quantise/dequantise, returned in the original [R, C] orientation."""
    c, s = quantize_colwise_t(a)
    return dequantize_rowwise(c, s).T
