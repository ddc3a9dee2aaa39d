"""Pins of the dequantised weight's rounding, against values fixed outside the oracle.

QLoRA explainer, "The QLoRA recipe: quantize, then adapt", stage 3: each frozen block is turned back
into bf16 before it is multiplied by the input.  The readings this file pins (listed with the other
readings of the pages in the design notes):

  NF-k (QLoRA "Innovation 1" and "Innovation 2"):  bf16( fp32(level) * fp32( fp32(E4M3(c1_8)) * s2 ) )
  INT4 group (QA-LoRA abstract, group-wise INT4):  bf16( fp32( fp32(code - z) * scale ) )

Every case puts the fp32 product exactly on a bf16 rounding tie or one fp32 ulp to either side of one,
so a dropped final rounding, a truncation instead of round-to-nearest-even, the two multiplications of
the NF-k path taken in the other order, the product taken in fp16 or in fp64 all move the answer.  The
expected bf16 bit patterns are literals; the test also re-derives each of them with exact rational
arithmetic (fractions.Fraction) and an IEEE round-to-nearest-even written here from its definition,
independently of numpy's floating point.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import quantize as Q
from oracle.codebook import nf_codebook_f32


def _rne(x: Fraction, sig: int) -> Fraction:
    """Round x to `sig` significant bits, ties to even (normal numbers; enough for these cases)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a, e = abs(x), 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    m = a * 2 ** (sig - 1)
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * Fraction(fl) * Fraction(2) ** (e - (sig - 1))


def _f32(x):
    return _rne(x, 24)


def _bf16_bits(x: Fraction) -> int:
    v = _rne(x, 8)
    return int(np.array([np.float32(float(v))]).view(np.uint32)[0] >> 16)


def _u32_to_frac(u: int) -> Fraction:
    return Fraction(float(np.array([u], np.uint32).view(np.float32)[0]))


def _u16_fp16_to_frac(u: int) -> Fraction:
    return Fraction(float(np.array([u], np.uint16).view(np.float16)[0]))


def _e4m3_frac(b: int) -> Fraction:
    """Value of an E4M3 byte (normal encodings only), from the format's definition: bias 7, 3 mantissa bits."""
    e, m = (b >> 3) & 0xF, b & 0x7
    assert 0 < e and (b & 0x7F) != 0x7F
    return (-1 if b & 0x80 else 1) * Fraction(8 + m, 8) * Fraction(2) ** (e - 7)


# fp32 bit patterns of the NF4 levels used below (the quantile construction's levels rounded to fp32)
NF4_LEVEL_BITS = {0: 0xBF800000, 3: 0xBECA329E, 6: 0xBDBA7869, 9: 0x3E24CADF, 12: 0x3EE1A4B5, 14: 0x3F3913B0,
                  15: 0x3F800000}

# (level index, E4M3 byte of c1_8, fp32 bits of s2, expected bf16 bits, where the fp32 product sits)
NF4_CASES = [
    (0, 0x36, 0x395E4924, 0xB942, "tie, rounds to even (down)"),
    (0, 0x36, 0x395E4926, 0xB943, "one fp32 ulp above a tie"),
    (0, 0x36, 0x395E4923, 0xB942, "one fp32 ulp below a tie"),
    (0, 0x7E, 0x39276DB7, 0xBD92, "tie; the exact product rounds the other way"),
    (3, 0x5B, 0x3940E7DB, 0xBAD2, "one fp32 ulp above a tie; the exact product rounds the other way"),
    (6, 0x36, 0x39868A9F, 0xB7AB, "one fp32 ulp below a tie; the other multiplication order rounds the other way"),
    (6, 0x5B, 0x394F2DCE, 0xB9D0, "tie; the exact product rounds the other way"),
    (9, 0x7E, 0x3961EB36, 0x3C7E, "tie; the exact product rounds the other way"),
    (12, 0x36, 0x394323C9, 0x3897, "one fp32 ulp above a tie; the other multiplication order rounds the other way"),
    (12, 0x5B, 0x39839B1C, 0x3B20, "tie, rounds to even (up)"),
    (12, 0x5B, 0x39839B1B, 0x3B1F, "one fp32 ulp below a tie"),
    (14, 0x36, 0x39549E74, 0x3907, "one fp32 ulp above a tie; the other multiplication order rounds the other way"),
    (14, 0x7E, 0x394E4BB4, 0x3D83, "one fp32 ulp above a tie; the other multiplication order rounds the other way"),
    (15, 0x5B, 0x39391746, 0x3B7E, "tie; the exact product rounds the other way"),
    (15, 0x7E, 0x39804925, 0x3DE1, "one fp32 ulp above a tie"),
]

# (code, fp16 bits of z, fp16 bits of scale, expected bf16 bits, where the product sits)
INT4_CASES = [
    (1, 0x0000, 0x2004, 0x3C00, "(c - z) s is a bf16 tie that rounds to even (down)"),
    (3, 0x0000, 0x2008, 0x3CC2, "(c - z) s is a bf16 tie that rounds to even (up)"),
    (0, 0x3C00, 0x2004, 0xBC00, "negative tie"),
    (0, 0x4200, 0x2003, 0xBCC1, "a product an fp16 rounding would move onto a tie"),
    (11, 0x3D4D, 0x2785, 0x3E92, "merged (non-integer) zero point: the fp32 rounding of the product decides"),
]


def _nf_q(level_idx, e4m3, s2_bits):
    codes = np.full(64, level_idx, np.uint8)
    return {"codes": codes, "bits": 4, "block": 64, "dq_block": 256, "c1_fp8": np.array([e4m3], np.uint8),
            "s2": np.array([s2_bits], np.uint32).view(np.float32), "shape": (1, 64)}


def test_nf4_level_literals():
    lev = nf_codebook_f32(4).view(np.uint32)
    for i, bits in NF4_LEVEL_BITS.items():
        assert int(lev[i]) == bits, i


@pytest.mark.parametrize("idx,e4m3,s2_bits,want,where", NF4_CASES, ids=[f"nf{i}" for i in range(len(NF4_CASES))])
def test_nf_dequant_rounding(idx, e4m3, s2_bits, want, where):
    level = _u32_to_frac(NF4_LEVEL_BITS[idx])
    scale = _f32(_e4m3_frac(e4m3) * _u32_to_frac(s2_bits))
    assert _bf16_bits(_f32(level * scale)) == want, where          # the literal, re-derived exactly
    got = Q.dequant_nfk(_nf_q(idx, e4m3, s2_bits))
    assert got.dtype == np.float32
    bits = got.reshape(-1).view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "not a bf16 value"
    assert np.all(bits >> 16 == want), (where, hex(int(bits[0] >> 16)), hex(want))


def test_nf_dequant_cases_cover_every_mistake():
    """The table itself separates the alternatives: each plausible misreading gives another answer on some case."""
    alt_order = exact = trunc = 0
    for idx, e4m3, s2_bits, want, _ in NF4_CASES:
        lv, e8, s2 = _u32_to_frac(NF4_LEVEL_BITS[idx]), _e4m3_frac(e4m3), _u32_to_frac(s2_bits)
        alt_order += _bf16_bits(_f32(_f32(lv * e8) * s2)) != want
        exact += _bf16_bits(lv * e8 * s2) != want
        v = _f32(lv * _f32(e8 * s2))
        trunc += int(np.array([np.float32(float(v))]).view(np.uint32)[0] >> 16) != want
    assert alt_order >= 3 and exact >= 3 and trunc >= 3


@pytest.mark.parametrize("code,z_bits,sc_bits,want,where", INT4_CASES, ids=[f"int4_{i}" for i in range(len(INT4_CASES))])
def test_int4_dequant_rounding(code, z_bits, sc_bits, want, where):
    z, sc = _u16_fp16_to_frac(z_bits), _u16_fp16_to_frac(sc_bits)
    assert _bf16_bits(_f32(_f32(code - z) * sc)) == want, where
    q = {"codes": np.full(32, code, np.uint8), "group": 32, "shape": (1, 32),
         "scale": np.array([[sc_bits]], np.uint16).view(np.float16),
         "zero": np.array([[z_bits]], np.uint16).view(np.float16)}
    got = Q.dequant_int4_group(q)
    bits = got.reshape(-1).view(np.uint32)
    assert np.all(bits & 0xFFFF == 0), "not a bf16 value"
    assert np.all(bits >> 16 == want), (where, hex(int(bits[0] >> 16)), hex(want))
    # the merge path passes its zero points separately
    got2 = Q.dequant_int4_group({**q, "zero": np.zeros((1, 1), np.float16)}, zero=q["zero"])
    assert np.all(got2.reshape(-1).view(np.uint32) >> 16 == want)


def test_int4_dequant_cases_cover_every_mistake():
    fp16_product = exact = 0
    for code, z_bits, sc_bits, want, _ in INT4_CASES:
        z, sc = _u16_fp16_to_frac(z_bits), _u16_fp16_to_frac(sc_bits)
        fp16_product += _bf16_bits(_rne((code - z) * sc, 11)) != want
        exact += _bf16_bits((code - z) * sc) != want
    assert fp16_product >= 1 and exact >= 1
