"""Number formats used by the layer: bf16, fp16 and OCP FP8 E4M3 (oracle; test infrastructure).

* bf16: the compute dtype of the dequantised weights and the adapters
  (QLoRA explainer, "The QLoRA recipe: quantize, then adapt", stages 2 and 3).
* E4M3: the "8-bit floats" that hold the first-level constants after double
  quantisation (QLoRA explainer, "Innovation 2: Double Quantization").  The page
  does not name the 8-bit format; this oracle reads it as OCP FP8 E4M3 (bias 7,
  no infinities, largest finite 448, S.1111.111 is NaN), rounded to nearest with
  ties to even and saturated to the largest finite value.
* fp16: the QA-LoRA scale and zero point (group-wise INT4 with fp16 scale/zero).
"""
from __future__ import annotations

import numpy as np


def bf16_rn(x) -> np.ndarray:
    """fp32 -> bf16 with round-to-nearest-even; returns the bf16 values as fp32.

    Written from the definition: keep the top 16 bits of the fp32 pattern after
    adding half an ulp of the kept part (plus the kept lsb, for ties to even).
    NaN stays NaN.
    """
    a = np.ascontiguousarray(x, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)).astype(np.uint32)
    out = r.view(np.float32).copy()
    nan = np.isnan(a)
    out[nan] = np.float32("nan")
    return out


def bf16_bits(x) -> np.ndarray:
    """bf16 bit patterns (uint16) of values already representable in bf16."""
    a = np.ascontiguousarray(x, dtype=np.float32)
    return (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32)


def fp16_rn(x) -> np.ndarray:
    """Round fp32 or fp64 values to fp16 (numpy's conversion: one rounding, ties to even)."""
    return np.asarray(x).astype(np.float16)


# ---- OCP FP8 E4M3 -------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes) -> np.ndarray:
    """Value of each E4M3 byte as fp64 (NaN for 0x7F / 0xFF)."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (8 + m) * np.exp2(e.astype(np.float64) - 10.0))
    val = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


_POS_VALUES = e4m3_decode(np.arange(0, 127))  # codes 0..126, strictly increasing, 0 .. 448


def e4m3_encode(x) -> np.ndarray:
    """fp32 -> E4M3 byte, round to nearest, ties to the even code, saturating to +-448.

    Nearest is decided exactly in fp64 (every fp32 input and every E4M3 value is
    exact in fp64).  Non-finite input is rejected: the quantiser never produces it.
    """
    a = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(a)):
        raise ValueError("e4m3_encode: non-finite input")
    neg = np.signbit(a)
    mag = np.abs(a)
    hi = np.searchsorted(_POS_VALUES, mag, side="left")       # first value >= mag
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_hi = np.abs(_POS_VALUES[hi] - mag)
    d_lo = np.abs(mag - _POS_VALUES[lo])
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = (d_lo == d_hi) & (lo != hi)
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    pick = np.where(mag >= E4M3_MAX, 126, pick)
    return (pick | np.where(neg, 0x80, 0)).astype(np.uint8)
