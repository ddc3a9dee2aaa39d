"""Pins for the oracle's number formats (bf16, fp16, E4M3) against library routines and definitions."""
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle.numerics import bf16_rn, bf16_bits, bf16_from_bits, e4m3_decode, e4m3_encode, fp16_rn

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def test_bf16_rn_matches_torch_conversion():
    g = np.random.default_rng(1)
    x = np.concatenate([
        g.standard_normal(200_000).astype(np.float32) * np.float32(3.0),
        (g.standard_normal(10_000) * 1e-38).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.4e38, -3.4e38, 1.00390625, 1.01171875], np.float32),
    ])
    # exact ties: fp32 patterns whose low 16 bits are 0x8000
    ties = (g.integers(0x3F000000, 0x41000000, 1000, dtype=np.uint32) & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    x = np.concatenate([x, ties.view(np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(bf16_rn(x), ref)


def test_bf16_bits_round_trip():
    x = bf16_rn(np.linspace(-5, 5, 1001, dtype=np.float32))
    np.testing.assert_array_equal(bf16_from_bits(bf16_bits(x)), x)


def _fp16_exact_rne(v: float) -> float:
    """fp64 -> fp16 by exact rational arithmetic (normal range), ties to even."""
    f = Fraction(v)
    sign = -1 if f < 0 else 1
    a = abs(f)
    if a == 0:
        return 0.0
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -14)
    ulp = Fraction(2) ** (e - 10)
    q = a / ulp
    n = q.numerator // q.denominator
    rem = q - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * float(n * ulp)


def test_fp16_rn_single_rounding_from_fp64():
    g = np.random.default_rng(2)
    vals = list(g.uniform(-20, 20, 2000)) + list(g.uniform(-1e-3, 1e-3, 500))
    # values that sit just beside an fp16 halfway point (double rounding through fp32 would fail)
    base = np.float16(3.0)
    half_ulp = 2.0 ** -10 * 2 / 2
    vals += [float(base) + half_ulp * 0.5 + 2.0 ** -40, float(base) + 2.0 ** -10 * 0.5 + 2.0 ** -30,
             7.5 + 2.0 ** -9 + 2.0 ** -35]
    for v in vals:
        assert float(fp16_rn(np.float64(v))) == _fp16_exact_rne(v), v


def test_e4m3_decode_spot_values():
    d = e4m3_decode(np.arange(256))
    assert d[0x00] == 0.0
    assert d[0x01] == 2.0 ** -9           # smallest subnormal
    assert d[0x07] == 7 * 2.0 ** -9
    assert d[0x08] == 2.0 ** -6           # smallest normal
    assert d[0x38] == 1.0
    assert d[0x39] == 1.125
    assert d[0x7E] == 448.0               # largest finite
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    assert d[0xB8] == -1.0
    assert np.all(np.diff(d[0:127]) > 0)  # monotone


def test_e4m3_round_trip_all_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    vals = e4m3_decode(codes).astype(np.float32)
    vals[codes == 0x80] = np.float32(-0.0)
    np.testing.assert_array_equal(e4m3_encode(vals), codes.astype(np.uint8))


def test_e4m3_ties_and_saturation():
    assert e4m3_encode(np.float32(1.0625)) == 0x38     # tie 1.0 / 1.125 -> even code
    assert e4m3_encode(np.float32(1.1875)) == 0x3A     # tie 1.125 / 1.25 -> even code
    assert e4m3_encode(np.float32(2.0 ** -10)) == 0x00  # tie 0 / 2^-9 -> 0
    assert e4m3_encode(np.float32(448.0)) == 0x7E
    assert e4m3_encode(np.float32(460.0)) == 0x7E
    assert e4m3_encode(np.float32(1e6)) == 0x7E        # saturate, never NaN
    assert e4m3_encode(np.float32(-1e6)) == 0xFE


def test_e4m3_matches_torch_in_range():
    g = np.random.default_rng(3)
    x = np.concatenate([g.uniform(-448, 448, 100_000), g.uniform(-1, 1, 100_000),
                        g.uniform(-0.02, 0.02, 20_000)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(e4m3_encode(x), ref)
