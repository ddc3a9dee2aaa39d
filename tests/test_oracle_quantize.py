"""Pins for the quantisers, packing, dequantisation and merge: brute force on tiny
inputs, exact-arithmetic nearest levels, special cases and error bounds."""
from fractions import Fraction

import numpy as np
import pytest

from oracle.codebook import nf_codebook_f32, zero_index
from oracle.layer import f64, forward, pool, rel_fro
from oracle.numerics import bf16_rn, e4m3_decode
from oracle import quantize as Q
from synth import random_matrix, to_bf16_values

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def brute_nf_codes(W, bits, block):
    """Scalar loops: block absmax, fp32 division, fp32 distance, first minimum."""
    flat = [np.float32(v) for v in np.asarray(W, np.float32).reshape(-1)]
    levels = [np.float32(v) for v in nf_codebook_f32(bits)]
    while len(flat) % block:
        flat.append(np.float32(0))
    codes, c1s = [], []
    for b0 in range(0, len(flat), block):
        blk = flat[b0:b0 + block]
        c1 = np.float32(0)
        for v in blk:
            if abs(v) > c1:
                c1 = np.float32(abs(v))
        c1s.append(c1)
        for v in blk:
            if c1 == 0:
                codes.append(zero_index(bits))
                continue
            u = np.float32(v / c1)
            best, bi = None, None
            for i, q in enumerate(levels):
                d = np.float32(abs(np.float32(u - q)))
                if best is None or d < best:
                    best, bi = d, i
            codes.append(bi)
    return np.array(codes, np.uint8), np.array(c1s, np.float32)


@pytest.mark.parametrize("bits,block", [(4, 64), (4, 128), (3, 64), (2, 128)])
def test_nf_codes_brute_force(bits, block):
    W = random_matrix(5, bits, "W", (6, 64), 0.02)
    W[1, :] = 0.0                     # an all-zero block
    q = Q.quantize_nfk(W, bits, block, 256)
    codes, c1 = brute_nf_codes(W, bits, block)
    np.testing.assert_array_equal(q["codes"], codes)
    np.testing.assert_array_equal(q["c1"], c1)


def test_nf_codes_are_exact_nearest_levels():
    """The fp32 argmin equals the exact-arithmetic nearest level except where the two
    candidates' exact distances differ by less than the fp32 rounding of u - q."""
    W = random_matrix(6, 0, "W", (64, 1024), 0.02)
    q = Q.quantize_nfk(W, 4, 64, 0)
    lev = nf_codebook_f32(4).astype(np.float64)
    u = (W.reshape(-1, 64) / q["c1"][:, None]).astype(np.float32).astype(np.float64).reshape(-1)
    exact = np.argmin(np.abs(u[:, None] - lev[None, :]), axis=1)
    diff = np.flatnonzero(exact != q["codes"])
    for i in diff:
        a, b = abs(u[i] - lev[exact[i]]), abs(u[i] - lev[q["codes"][i]])
        assert abs(a - b) <= 2.0 ** -24 * 2
    assert diff.size <= 5


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_nf_special_cases(bits):
    lev = nf_codebook_f32(bits)
    n = 64
    row = np.zeros(n, np.float32)
    row[: lev.size] = lev            # absmax is exactly 1 -> u == level
    W = np.stack([row, np.zeros(n, np.float32), np.full(n, -3.0, np.float32)])
    W[2, 1] = 3.0
    q = Q.quantize_nfk(W, bits, 64, 0)
    codes = q["codes"].reshape(3, n)
    np.testing.assert_array_equal(codes[0, : lev.size], np.arange(lev.size))
    assert np.all(codes[1] == zero_index(bits))
    assert codes[2, 0] == 0 and codes[2, 1] == lev.size - 1     # -absmax, +absmax -> end codes


def test_nf_tie_takes_lowest_index():
    lev = nf_codebook_f32(4).astype(np.float64)
    found = 0
    for i in range(15):
        mid = (Fraction(float(lev[i])) + Fraction(float(lev[i + 1]))) / 2
        m32 = np.float32(float(mid))
        if Fraction(float(m32)) != mid:
            continue
        if np.float32(abs(np.float32(m32 - np.float32(lev[i])))) != np.float32(abs(np.float32(m32 - np.float32(lev[i + 1])))):
            continue
        W = np.zeros((1, 64), np.float32)
        W[0, 0] = 1.0
        W[0, 1] = m32
        q = Q.quantize_nfk(W, 4, 64, 0)
        assert q["codes"][1] == i
        found += 1
    # construct ties by hand if the levels give none: u exactly halfway in fp32
    W = np.zeros((1, 64), np.float32)
    W[0, 0] = 1.0
    a, b = np.float32(lev[7]), np.float32(lev[8])     # 0 and the first positive level
    m = np.float32(b / 2)
    W[0, 1] = m
    q = Q.quantize_nfk(W, 4, 64, 0)
    da = np.float32(abs(np.float32(m - a)))
    db = np.float32(abs(np.float32(m - b)))
    assert q["codes"][1] == (7 if da <= db else 8)


def test_double_quant_constants():
    W = random_matrix(7, 0, "W", (64, 64 * 300), 0.02)    # 300 blocks per row -> partial last group
    q = Q.quantize_nfk(W, 4, 64, 256)
    c1 = q["c1"]
    ng = -(-c1.size // 256)
    assert q["s2"].size == ng
    for g in range(ng):
        seg = c1[g * 256:(g + 1) * 256]
        assert q["s2"][g] == np.float32(seg.max() / np.float32(448))
        dec = e4m3_decode(q["c1_fp8"][g * 256:(g + 1) * 256]) * q["s2"][g]
        np.testing.assert_allclose(dec, seg, rtol=2.0 ** -4 + 1e-6)
        assert q["c1_fp8"][g * 256 + int(np.argmax(seg))] == 0x7E    # group max -> 448


def test_double_quant_zero_group():
    c1 = np.zeros(300, np.float32)
    c1[260] = 0.5
    c8, s2 = Q.double_quantize(c1, 256)
    assert s2[0] == 0 and np.all(c8[:256] == 0)
    assert c8[260] == 0x7E


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_packing_bit_layout(bits):
    g = np.random.default_rng(bits)
    codes = g.integers(0, 2 ** bits, 96, dtype=np.uint8)
    packed = Q.pack_codes(codes, bits)
    assert packed.size == 96 * bits // 8
    bitstr = []
    if bits == 4:
        for j in range(48):
            byte = 0
            for bit in range(4):
                byte |= ((int(codes[2 * j]) >> bit) & 1) << bit
                byte |= ((int(codes[2 * j + 1]) >> bit) & 1) << (4 + bit)
            bitstr.append(byte)
    elif bits == 2:
        for j in range(24):
            byte = 0
            for t in range(4):
                byte |= int(codes[4 * j + t]) << (2 * t)
            bitstr.append(byte)
    else:
        for grp in range(3):
            for p in range(3):
                word = 0
                for t in range(32):
                    word |= ((int(codes[32 * grp + t]) >> p) & 1) << t
                bitstr += [(word >> (8 * i)) & 0xFF for i in range(4)]
    np.testing.assert_array_equal(packed, np.array(bitstr, np.uint8))
    np.testing.assert_array_equal(Q.unpack_codes(packed, bits, 96), codes)


@pytest.mark.parametrize("bits,block,dq", [(4, 64, 256), (4, 64, 0), (3, 128, 256), (2, 64, 256)])
def test_nf_dequant_error_bound(bits, block, dq):
    W = random_matrix(8, bits, "W", (32, 512), 0.02)
    q = Q.quantize_nfk(W, bits, block, dq)
    Wd = Q.dequant_nfk(q)
    lev = nf_codebook_f32(bits).astype(np.float64)
    halfgap = np.max(np.diff(lev)) / 2
    c1 = np.repeat(q["c1"], block)[: W.size].reshape(W.shape).astype(np.float64)
    sc = np.repeat(Q.nf_block_scales(q), block)[: W.size].reshape(W.shape).astype(np.float64)
    # the block scale is c1 itself, or with double quantisation c1 to E4M3 precision: a relative
    # error of at most 2^-4 in the normal range, half the subnormal spacing (2^-10 s2) below it
    if dq:
        s2 = np.repeat(np.repeat(q["s2"], dq)[: q["c1"].size], block)[: W.size].reshape(W.shape).astype(np.float64)
        scale_err = c1 * 2.0 ** -4 * (1 + 1e-6) + s2 * 2.0 ** -10
        assert np.all(np.abs(sc - c1) <= scale_err)
    else:
        scale_err = np.zeros_like(c1)
        np.testing.assert_array_equal(sc, c1)
    # |level| <= 1, so the scale's error moves a value by at most scale_err
    bound = c1 * halfgap * (1 + 1e-6) + scale_err + np.abs(Wd) * 2.0 ** -8
    assert np.all(np.abs(W - Wd) <= bound)
    # dequant is level * scale rounded to bf16, level taken from the code
    ref = bf16_rn((nf_codebook_f32(bits)[q["codes"][: W.size]] * sc.reshape(-1).astype(np.float32)).astype(np.float32))
    np.testing.assert_array_equal(Wd.reshape(-1), ref)


def test_int4_group_properties():
    W = random_matrix(9, 0, "W", (16, 256), 0.02)
    W[0, :32] = 0.0                     # degenerate group
    W[1, 32:64] = np.abs(W[1, 32:64])   # all non-negative group: lo = 0 -> z = 0
    q = Q.quantize_int4_group(W, 32)
    sc = q["scale"].astype(np.float32)
    z = q["zero"].astype(np.float32)
    assert sc[0, 0] == 0 and z[0, 0] == 0 and np.all(q["codes"].reshape(16, 256)[0, :32] == 0)
    assert z[1, 1] == 0
    assert q["zero"].view(np.uint16)[1, 1] == 0          # an integer zero point: +0, not -0
    assert np.all((z >= 0) & (z <= 15) & (z == np.rint(z)))
    codes = q["codes"].reshape(16, 8, 32).astype(np.float64)
    assert codes.max() <= 15
    rec = (codes - z[..., None]) * sc[..., None]
    err = np.abs(rec - W.reshape(16, 8, 32))
    assert np.all(err <= sc[..., None].astype(np.float64) * 0.51 + 1e-12)
    g = W.reshape(16, 8, 32).astype(np.float64)
    span = np.maximum(g.max(-1), 0) - np.minimum(g.min(-1), 0)
    np.testing.assert_allclose(sc[sc > 0], (span / 15)[sc > 0], rtol=2.0 ** -10)


def test_int4_group_brute_force_tiny():
    W = random_matrix(10, 0, "W", (3, 64), 0.02)
    q = Q.quantize_int4_group(W, 32)
    for o in range(3):
        for g in range(2):
            grp = [np.float32(v) for v in W[o, 32 * g:32 * g + 32]]
            lo = min(np.float32(0), min(grp))
            hi = max(np.float32(0), max(grp))
            scale = np.float16(np.float32(np.float32(hi - lo) / np.float32(15)))
            sf = np.float32(scale)
            assert q["scale"][o, g] == scale
            z = float(np.clip(np.rint(np.float32(-lo / sf)), 0, 15))
            assert float(q["zero"][o, g]) == z
            for j, v in enumerate(grp):
                t = np.float32(np.float32(v / sf) + np.float32(z))
                c = int(np.clip(np.rint(t), 0, 15))
                assert q["codes"][o * 64 + 32 * g + j] == c


def test_qalora_merge_is_lossless_in_fp64():
    """Merged and unmerged outputs agree (fp64, unrounded z'): QA-LoRA's abstract says the merge loses no accuracy."""
    N, K, L, r, M, s = 64, 256, 32, 4, 8, 1.5
    W = random_matrix(11, 0, "W", (N, K), 0.02)
    A = random_matrix(11, 1, "A", (r, K // L), 0.01, bf16=True)
    B = random_matrix(11, 2, "B", (N, r), 0.01, bf16=True)
    X = random_matrix(11, 3, "X", (M, K), 1.0, bf16=True)
    q = Q.quantize_int4_group(W, L)
    sc = q["scale"].astype(np.float64)
    codes = q["codes"].reshape(N, K // L, L).astype(np.float64)
    Wq = ((codes - q["zero"].astype(np.float64)[..., None]) * sc[..., None]).reshape(N, K)
    unmerged = forward(X, Wq, A, B, s, L=L)["Y"]
    zp = Q.qalora_merged_zero_fp64(q, A, B, s)
    Wm = ((codes - zp[..., None]) * sc[..., None]).reshape(N, K)
    merged = f64(X) @ Wm.T
    assert rel_fro(merged, unmerged) < 1e-12
    # with the stored fp16 z' and the bf16 dequant the two stay within the bf16 tolerance
    zp16 = Q.qalora_merge(q, A, B, s)
    merged16 = f64(X) @ Q.dequant_int4_group(q, zero=zp16).astype(np.float64).T
    assert rel_fro(merged16, unmerged) < 1e-2


def test_int4_exact_halves_round_to_even():
    # scale 0.0625 exactly (span 0.9375 = 15 x 0.0625); values at k + 1/2 steps are fp32-exact ties
    s = 0.0625
    W = np.zeros((2, 32), np.float32)
    W[0, :5] = [15 * s, 0.5 * s, 1.5 * s, 2.5 * s, 3.5 * s]           # lo = 0 -> z = 0
    W[1, :4] = [-2.5 * s, 12.5 * s, 0.5 * s, 1.5 * s]                 # -lo / scale = 2.5 -> z = 2
    q = Q.quantize_int4_group(W, 32)
    assert np.all(q["scale"].astype(np.float32) == np.float32(s))
    assert float(q["zero"][0, 0]) == 0.0 and float(q["zero"][1, 0]) == 2.0
    codes = q["codes"].reshape(2, 32)
    assert list(codes[0, :5]) == [15, 0, 2, 2, 4]                      # 0.5 -> 0, 1.5 -> 2, 2.5 -> 2, 3.5 -> 4
    assert list(codes[1, :4]) == [0, 14, 2, 4]                         # -0.5 -> 0, 14.5 -> 14, 2.5 -> 2, 3.5 -> 4


def test_qalora_merge_rounds_once_from_fp64():
    # z' = 2 - a / 32 = 1 + 2^-11 + 2^-30: one rounding to fp16 goes up to 1 + 2^-10; rounding through
    # fp32 first would land on the tie 1 + 2^-11 and then round to even, 1
    a = 32.0 - 2.0 ** -6 - 2.0 ** -25
    q = {"group": 32, "scale": np.array([[1.0]], np.float16), "zero": np.array([[2.0]], np.float16)}
    zp = Q.qalora_merge(q, np.array([[a]]), np.array([[1.0]]), 1.0)
    assert float(zp[0, 0]) == 1.0 + 2.0 ** -10


def test_nf_partial_last_block_is_zero_padded():
    W = random_matrix(12, 0, "W", (1, 192), 0.02)     # block 128: the second block has 64 weights
    q = Q.quantize_nfk(W, 4, 128, 0)
    assert q["c1"][1] == np.float32(np.abs(W[0, 128:]).max())
    assert np.all(q["codes"][192:] == zero_index(4))   # the padding takes the zero level
