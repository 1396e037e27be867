"""Pins for the oracle's MXFP8 codec and block quantiser (CPU only).

The pages fix only "8 bits per value, one scale per block of 32 values"
("MoE-Training für biologische Grundmodelle optimieren", hyper.ai/de, MXFP8
passage). E4M3/E8M0 and the scale rule are the OCP MX reading; these tests pin the
oracle against that format's closed-form facts and hand-derived blocks."""
import math
import os

import numpy as np
import pytest

from oracle import mxfp8

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mxfp8_blocks.txt")


def _parse_value(s):
    s = s.strip()
    if "*2^" in s:
        p, q = s.split("*2^")
        return float(p) * math.ldexp(1.0, int(q))
    return float(s)


def _golden_blocks():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        name, vals, scale, codes = [f.strip() for f in line.split("|")]
        v = np.zeros(32)
        for item in vals.split(","):
            pos, val = item.split(":")
            v[int(pos)] = _parse_value(val)
        exp_codes = {int(p): int(c, 16) for p, c in (it.split(":") for it in codes.split(","))}
        out.append((name, v, int(scale, 16), exp_codes))
    return out


@pytest.mark.parametrize("name,v,scale,codes", _golden_blocks(), ids=lambda x: x if isinstance(x, str) else "")
def test_hand_built_blocks(name, v, scale, codes):
    q, s = mxfp8.quantize_blocks(v[None, :])
    assert int(s[0]) == scale, name
    for pos, c in codes.items():
        assert int(q[0, pos]) == c, (name, pos, hex(int(q[0, pos])), hex(c))


def test_decode_closed_form_points():
    assert mxfp8.e4m3_decode(0x7E) == 448.0
    assert mxfp8.e4m3_decode(0xFE) == -448.0
    assert mxfp8.e4m3_decode(0x78) == 256.0
    assert mxfp8.e4m3_decode(0x38) == 1.0
    assert mxfp8.e4m3_decode(0x08) == 2.0 ** -6        # smallest normal
    assert mxfp8.e4m3_decode(0x07) == 7 * 2.0 ** -9    # largest subnormal
    assert mxfp8.e4m3_decode(0x01) == 2.0 ** -9        # smallest subnormal
    assert mxfp8.e4m3_decode(0x00) == 0.0
    assert math.copysign(1.0, mxfp8.e4m3_decode(0x80)) == -1.0
    assert np.isnan(mxfp8.e4m3_decode(0x7F)) and np.isnan(mxfp8.e4m3_decode(0xFF))


def test_decode_monotone_and_count():
    vals = mxfp8.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(vals) > 0)
    allv = mxfp8.e4m3_decode(np.arange(256))
    assert np.sum(np.isfinite(allv)) == 254


def test_exhaustive_round_trip():
    """Every finite code, placed in a block whose amax is 448 (scale exponent 0),
    re-encodes to itself."""
    for b in range(256):
        if b in (0x7F, 0xFF):
            continue
        v = np.zeros(32)
        v[0] = 448.0
        v[1] = mxfp8.e4m3_decode(b)
        q, s = mxfp8.quantize_blocks(v[None, :])
        assert s[0] == 127
        assert q[0, 1] == b, hex(b)


def test_encode_midpoints_round_to_even():
    """Between every pair of neighbouring codes, the midpoint goes to the even code and
    points just either side go to the nearer one."""
    vals = mxfp8.e4m3_decode(np.arange(0x7F))
    for c in range(0x7E):
        lo, hi = vals[c], vals[c + 1]
        mid = 0.5 * (lo + hi)
        want = c if c % 2 == 0 else c + 1
        assert mxfp8.e4m3_encode(mid) == want
        eps = (hi - lo) * 1e-3
        assert mxfp8.e4m3_encode(mid - eps) == c
        assert mxfp8.e4m3_encode(mid + eps) == c + 1


def test_scale_exponent_rule():
    for a in [1e-30, 2.0 ** -126, 0.3, 1.0, 1.999, 2.0, 447.0, 448.0, 1e30]:
        want = max(-127, min(127, math.floor(math.log2(a)) - 8))
        assert mxfp8.scale_exponent(a) == want
    assert mxfp8.scale_exponent(0.0) == -127
    assert mxfp8.scale_exponent(2.0 ** 200) == 127


def test_quantisation_error_bound():
    """Relative error of a dequantised element is at most 2^-4 (half an ulp of a 3-bit
    mantissa) wherever the scaled value lies in E4M3's normal, unsaturated range."""
    rng = np.random.default_rng(0)
    v = rng.standard_normal((500, 32)) * np.exp2(rng.integers(-20, 20, (500, 1)))
    q, s = mxfp8.quantize_blocks(v)
    d = mxfp8.dequantize_blocks(q, s)
    X = s.astype(np.int64) - 127
    lo = np.exp2(X - 6.0)[:, None]
    hi = 448.0 * np.exp2(X.astype(float))[:, None]
    normal = (np.abs(v) >= lo) & (np.abs(v) <= hi)      # not subnormal, not saturated
    rel = np.abs(d - v)[normal] / np.abs(v)[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-15
    # and the block max never exceeds 448 * 2^X
    assert np.all(np.abs(d) <= 448.0 * np.exp2(X.astype(float))[:, None])


def test_rowwise_and_colwise_shapes():
    rng = np.random.default_rng(1)
    a = rng.standard_normal((64, 96))
    c, s = mxfp8.quantize_rowwise(a)
    assert c.shape == (64, 96) and s.shape == (64, 3)
    ct, st = mxfp8.quantize_colwise_t(a)
    assert ct.shape == (96, 64) and st.shape == (96, 2)
    # colwise of a == rowwise of a^T, block by block
    np.testing.assert_array_equal(ct, mxfp8.quantize_rowwise(a.T)[0])
    # each colwise block covers 32 consecutive rows of one column
    blk = a[32:64, 5]
    qb, sb = mxfp8.quantize_blocks(blk[None, :])
    np.testing.assert_array_equal(ct[5, 32:64], qb[0])
    assert st[5, 1] == sb[0]


# ----------------------------------------------------------------------------- E5M2 (gradient variant)

def _fp16_of_e5m2_code(c):
    """E5M2 is the high byte of IEEE binary16 (same sign, 5-bit exponent with bias 15,
    top 2 mantissa bits): an independent decoder through numpy's float16."""
    return np.array([c << 8], dtype=np.uint16).view(np.float16).astype(np.float64)[0]


def test_e5m2_decode_is_fp16_high_byte():
    for c in range(256):
        want = _fp16_of_e5m2_code(c)
        got = float(mxfp8.e5m2_decode(c))
        if np.isnan(want):
            assert np.isnan(got), hex(c)
        else:
            assert got == want and math.copysign(1.0, got) == math.copysign(1.0, want), hex(c)
    assert mxfp8.e5m2_decode(0x7B) == 57344.0 == mxfp8.E5M2_MAX
    assert mxfp8.e5m2_decode(0x04) == 2.0 ** -14         # smallest normal
    assert mxfp8.e5m2_decode(0x01) == 2.0 ** -16         # smallest subnormal
    assert mxfp8.e5m2_decode(0x3C) == 1.0


def test_e5m2_encode_matches_fp16_integer_rounding():
    """For every value representable in binary16 with |v| <= 57344, the nearest-even E5M2
    code is the fp16 bit pattern rounded to its high byte with round-half-to-even on the
    integer bits (IEEE rounding carries across the subnormal/normal boundary)."""
    bits = np.arange(0, 0x7C00, dtype=np.uint32)            # all finite non-negative fp16
    v = bits.astype(np.uint16).view(np.float16).astype(np.float64)
    keep = v <= 57344.0
    bits, v = bits[keep], v[keep]
    want = ((bits + 0x7F + ((bits >> 8) & 1)) >> 8).astype(np.uint8)
    got = mxfp8.e5m2_encode(v)
    assert np.array_equal(got, want)
    assert np.array_equal(mxfp8.e5m2_encode(-v[1:]), want[1:] | 0x80)


def test_e5m2_saturates_instead_of_infinity():
    v = np.zeros(32)
    v[0] = 65535.0                                         # amax < 2^16: X = 0
    v[1] = 61440.0                                         # IEEE would round to infinity
    q, s = mxfp8.quantize_blocks(v[None, :], "e5m2")
    assert s[0] == 127 and q[0, 0] == 0x7B and q[0, 1] == 0x7B


def test_e5m2_scale_rule_and_error_bound():
    for a in [1e-30, 0.3, 1.0, 2.0, 57344.0, 65535.0, 1e30]:
        want = max(-127, min(127, math.floor(math.log2(a)) - 15))
        assert mxfp8.scale_exponent(a, mxfp8.E5M2_EMAX) == want
    rng = np.random.default_rng(3)
    v = rng.standard_normal((500, 32)) * np.exp2(rng.integers(-20, 20, (500, 1)))
    q, s = mxfp8.quantize_blocks(v, "e5m2")
    d = mxfp8.dequantize_blocks(q, s, "e5m2")
    X = (s.astype(np.int64) - 127).astype(float)[:, None]
    normal = (np.abs(v) >= np.exp2(X - 14.0)) & (np.abs(v) <= 57344.0 * np.exp2(X))
    rel = np.abs(d - v)[normal] / np.abs(v)[normal]
    assert rel.max() <= 2.0 ** -3 + 1e-15                   # half an ulp of a 2-bit mantissa
    assert rel.max() > 2.0 ** -4                            # coarser than E4M3
    # a block quantised to E5M2 keeps 6 more binades below its max than E4M3
    assert np.all(np.abs(d) <= 57344.0 * np.exp2(X))


# ----------------------------------------------------------------------------- "ceil" scale rule (variant)

@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_ceil_rule_is_the_smallest_non_saturating_power_of_two(fmt):
    """Brute force over candidate exponents: the ceil rule picks the smallest X for which
    amax * 2^-X does not exceed the format's largest value; the OCP rule picks X or X - 1."""
    _, decode, emax, vmax = mxfp8.FORMATS[fmt]
    rng = np.random.default_rng(7)
    amax = np.abs(rng.standard_normal(2000)) * np.exp2(rng.integers(-60, 60, 2000))
    amax = np.concatenate([amax, vmax * np.exp2(np.arange(-20.0, 20.0)),          # exactly at the top: no +1
                           np.nextafter(vmax, np.inf) * np.exp2(np.arange(-20.0, 20.0))])  # just above: +1
    Xc = mxfp8.scale_exponent(amax, emax, "ceil", vmax)
    Xo = mxfp8.scale_exponent(amax, emax)
    for a, xc, xo in zip(amax, Xc, Xo):
        cands = [x for x in range(-127, 128) if a <= vmax * 2.0 ** x]
        assert xc == min(cands), (a, xc)
        assert xc - xo in (0, 1)
    assert np.all(Xc[-40:] == Xo[-40:] + 1) and np.all(Xc[-80:-40] == Xo[-80:-40])


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_ceil_rule_never_saturates(fmt):
    """Under the ceil rule no element of a block reaches beyond the format's top value, and
    a block whose amax the OCP rule would saturate gets the next scale up."""
    _, decode, _, vmax = mxfp8.FORMATS[fmt]
    rng = np.random.default_rng(8)
    v = rng.standard_normal((400, 32)) * np.exp2(rng.integers(-30, 30, (400, 1)))
    q, s = mxfp8.quantize_blocks(v, fmt, "ceil")
    X = (s.astype(np.int64) - 127).astype(float)[:, None]
    assert np.all(np.abs(v) * np.exp2(-X) <= vmax)
    d = mxfp8.dequantize_blocks(q, s, fmt)
    rel = np.abs(d - v)[np.abs(v) * np.exp2(-X) >= 1.0] / np.abs(v)[np.abs(v) * np.exp2(-X) >= 1.0]
    assert rel.max() <= (2.0 ** -4 if fmt == "e4m3" else 2.0 ** -3) + 1e-15
    blk = np.zeros(32)
    blk[0] = 480.0 if fmt == "e4m3" else 60000.0        # saturates under the OCP rule
    q4, s4 = mxfp8.quantize_blocks(blk[None, :], fmt)
    qc, sc = mxfp8.quantize_blocks(blk[None, :], fmt, "ceil")
    assert decode(q4[0, 0]) == vmax and sc[0] == s4[0] + 1
    back = decode(qc[0, 0]) * 2.0 ** (int(sc[0]) - 127)
    if fmt == "e4m3":
        assert back == blk[0]                 # 480 = 240 * 2, and 240 is an E4M3 value
    else:
        assert abs(back - blk[0]) <= 2.0 ** -3 * blk[0]   # rounded, not clipped to 57344
