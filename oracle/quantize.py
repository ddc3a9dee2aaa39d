"""Quantisers, packing, dequantisation and the QA-LoRA merge (oracle; test infrastructure).

NF-k blockwise quantisation follows the QLoRA explainer: "Background: what is
quantization?" (divide by the absolute maximum, round to the nearest level),
"Innovation 1: 4-bit NormalFloat (NF4)" (the levels), the page's code sketch
(absmax per block of 64 consecutive weights of the row-major flattened matrix,
argmin of |w/absmax - level|, first index on ties as numpy's argmin does, dequant
= level[code] * absmax), and "Innovation 2: Double Quantization" (the fp32
first-level constants, in groups of 256, become 8-bit floats with one fp32
second-level constant per group).

Readings where the pages leave a step open (each is listed in the design notes):
  * w / absmax is one fp32 IEEE division, rounded to nearest; distances
    |u - level| are fp32; the code is the first index of the minimum.
  * absmax == 0 (an all-zero block): every code is the index of the zero level.
  * codes are computed against the exact fp32 absmax; double quantisation is
    applied to the constants afterwards.
  * double quantisation: s2 = fp32(max(group) / 448); c1_8 = E4M3(fp32(c1 / s2));
    s2 == 0 gives c1_8 = 0.  No mean-centring.
  * a partial last block is padded with zeros; a partial last group uses the
    blocks it has.
  * packing (the pages give none; this layout is the contract):
      k=4  two codes per byte, element 2j in the low nibble, 2j+1 in the high nibble;
      k=2  four codes per byte, element 4j+t at bits 2t..2t+1;
      k=3  bit planes: every 32 consecutive codes form three little-endian uint32
           words, word p holding bit p of code t at bit t.
  * dequant: bf16_rn(fp32(level[code]) * (fp32(E4M3(c1_8)) * s2)), multiplications
    in that order, each rounded to fp32; without double quantisation
    bf16_rn(level[code] * c1).

QA-LoRA (abstract: group-wise INT4 quantisation, an adapter with fewer degrees of
freedom, and a merge into the quantised weight that costs no accuracy) is read as:
  * per (row o, group g of L consecutive inputs): lo = min(0, min w), hi = max(0, max w),
    scale = fp16_rn(fp32(fp32(hi - lo) / 15)), z = clamp(rne(fp32(-lo / scale)), 0, 15)
    stored as fp16 (an integer, so a zero is +0), code = clamp(rne(fp32(fp32(w / scale) + z)), 0, 15); a group whose
    fp16 scale is 0 has z = 0 and codes 0;
  * dequant = bf16_rn(fp32(fp32(code - z) * scale));
  * merge: the pooled adapter adds (s / L) (B A)[o, g] to every weight of group g of
    row o, which equals shifting the zero point:
        z'[o, g] = fp16_rn(z - s (B A)[o, g] / (L scale[o, g]))   in fp64.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from .codebook import nf_codebook_f32, zero_index
from .numerics import bf16_rn, e4m3_decode, e4m3_encode

_CHUNK = 1 << 18  # elements per argmin chunk (keeps the 2^k-wide distance tensor small)


def _check_finite(W: np.ndarray) -> None:
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")


# ---- NF-k --------------------------------------------------------------------------------

def nf_block_absmax(flat: np.ndarray, block: int) -> np.ndarray:
    nb = -(-flat.size // block)
    pad = np.zeros(nb * block, np.float32)
    pad[: flat.size] = flat
    return np.abs(pad.reshape(nb, block)).max(axis=1), pad.reshape(nb, block)


def nf_codes(blocks: np.ndarray, c1: np.ndarray, bits: int) -> np.ndarray:
    """First-index argmin over the levels of fp32 |fp32(w / c1) - level|; zero blocks -> zero level."""
    q = nf_codebook_f32(bits)
    nb, bl = blocks.shape
    codes = np.empty((nb, bl), np.uint8)
    rows_per_chunk = max(1, _CHUNK // bl)
    with np.errstate(divide="ignore", invalid="ignore"):
        for r0 in range(0, nb, rows_per_chunk):
            b = blocks[r0:r0 + rows_per_chunk]
            c = c1[r0:r0 + rows_per_chunk]
            u = b / c[:, None]                                  # fp32 / fp32 -> fp32 (RN)
            d = np.abs(u[:, :, None] - q[None, None, :])        # fp32
            idx = np.argmin(d, axis=-1).astype(np.uint8)        # first index on ties
            idx[c == 0] = zero_index(bits)
            codes[r0:r0 + rows_per_chunk] = idx
    return codes


def double_quantize(c1: np.ndarray, dq_block: int):
    """fp32 first-level constants -> (E4M3 bytes, fp32 second-level constants)."""
    nb = c1.size
    ng = -(-nb // dq_block)
    pad = np.zeros(ng * dq_block, np.float32)
    pad[:nb] = c1
    gmax = pad.reshape(ng, dq_block).max(axis=1)
    s2 = (gmax / np.float32(448.0)).astype(np.float32)
    s2_per_block = np.repeat(s2, dq_block)[:nb]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (c1 / s2_per_block).astype(np.float32)
    ratio = np.where(s2_per_block == 0, np.float32(0.0), ratio)
    return e4m3_encode(ratio), s2


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    c = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    if bits == 4:
        if c.size % 2:
            raise ValueError("k=4 packing needs an even count")
        return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)
    if bits == 2:
        if c.size % 4:
            raise ValueError("k=2 packing needs a multiple of 4")
        c4 = c.reshape(-1, 4).astype(np.uint8)
        return (c4[:, 0] | (c4[:, 1] << 2) | (c4[:, 2] << 4) | (c4[:, 3] << 6)).astype(np.uint8)
    if bits == 3:
        if c.size % 32:
            raise ValueError("k=3 packing needs a multiple of 32")
        g = c.reshape(-1, 32).astype(np.uint64)
        weights = (np.uint64(1) << np.arange(32, dtype=np.uint64))
        words = np.empty((g.shape[0], 3), np.uint32)
        for p in range(3):
            bitp = (g >> np.uint64(p)) & np.uint64(1)
            words[:, p] = (bitp * weights).sum(axis=1).astype(np.uint32)
        return words.reshape(-1).astype("<u4").view(np.uint8)
    raise ValueError("bits must be 2, 3 or 4")


def unpack_codes(packed: np.ndarray, bits: int, count: int) -> np.ndarray:
    p = np.ascontiguousarray(packed, dtype=np.uint8).reshape(-1)
    if bits == 4:
        out = np.empty(p.size * 2, np.uint8)
        out[0::2] = p & 0xF
        out[1::2] = p >> 4
        return out[:count]
    if bits == 2:
        out = np.empty(p.size * 4, np.uint8)
        for t in range(4):
            out[t::4] = (p >> (2 * t)) & 0x3
        return out[:count]
    if bits == 3:
        words = p.view("<u4").reshape(-1, 3).astype(np.uint64)
        t = np.arange(32, dtype=np.uint64)
        codes = np.zeros((words.shape[0], 32), np.uint64)
        for q in range(3):
            codes |= ((words[:, q:q + 1] >> t[None, :]) & np.uint64(1)) << np.uint64(q)
        return codes.reshape(-1).astype(np.uint8)[:count]
    raise ValueError("bits must be 2, 3 or 4")


def quantize_nfk(W: np.ndarray, bits: int = 4, block: int = 64, dq_block: int = 256) -> Dict[str, np.ndarray]:
    """Blockwise NF-k quantisation (+ double quantisation when dq_block > 0).

    Returns codes (unpacked, uint8, length = padded element count), packed bytes,
    c1 (fp32, one per block) and, with double quantisation, c1_fp8 (uint8) and s2 (fp32).
    """
    W = np.asarray(W, dtype=np.float32)
    _check_finite(W)
    flat = W.reshape(-1)
    c1, blocks = nf_block_absmax(flat, block)
    codes = nf_codes(blocks, c1, bits).reshape(-1)
    out = {"codes": codes, "packed": pack_codes(codes, bits), "c1": c1,
           "bits": bits, "block": block, "dq_block": dq_block, "shape": W.shape}
    if dq_block:
        c1_8, s2 = double_quantize(c1, dq_block)
        out["c1_fp8"] = c1_8
        out["s2"] = s2
    return out


def nf_block_scales(q: Dict[str, np.ndarray]) -> np.ndarray:
    """fp32 scale of every block: fp32(E4M3(c1_8)) * s2 with double quantisation, else c1."""
    if q["dq_block"]:
        nb = q["c1_fp8"].size
        s2b = np.repeat(q["s2"], q["dq_block"])[:nb]
        return (e4m3_decode(q["c1_fp8"]).astype(np.float32) * s2b).astype(np.float32)
    return q["c1"].astype(np.float32)


def dequant_nfk(q: Dict[str, np.ndarray]) -> np.ndarray:
    """bf16 values (as fp32) of the dequantised weight, shape of the original matrix."""
    levels = nf_codebook_f32(q["bits"])
    scales = nf_block_scales(q)
    block = q["block"]
    vals = levels[q["codes"]].reshape(-1, block) * scales[:, None]   # fp32 * fp32 -> fp32
    N, K = q["shape"]
    return bf16_rn(vals.reshape(-1)[: N * K]).reshape(N, K)


# ---- INT4 group-wise (QA-LoRA) -------------------------------------------------------------

def quantize_int4_group(W: np.ndarray, group: int = 32) -> Dict[str, np.ndarray]:
    W = np.asarray(W, dtype=np.float32)
    _check_finite(W)
    N, K = W.shape
    if K % group:
        raise ValueError("K must be a multiple of the group length")
    g = W.reshape(N, K // group, group)
    lo = np.minimum(np.float32(0.0), g.min(axis=-1))
    hi = np.maximum(np.float32(0.0), g.max(axis=-1))
    span = (hi - lo).astype(np.float32)
    scale16 = (span / np.float32(15.0)).astype(np.float32).astype(np.float16)
    scale = scale16.astype(np.float32)
    ok = scale > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        zf = np.rint((-lo / scale).astype(np.float32))
        # the zero point is an integer in [0, 15]; adding +0.0 maps a -0.0 (from lo == 0) to +0.0
        z = (np.where(ok, np.clip(zf, 0, 15), 0).astype(np.float32) + np.float32(0.0)).astype(np.float32)
        t = ((g / scale[..., None]).astype(np.float32) + z[..., None]).astype(np.float32)
        code = np.where(ok[..., None], np.clip(np.rint(t), 0, 15), 0).astype(np.uint8)
    codes = code.reshape(N, K)
    return {"codes": codes.reshape(-1), "packed": pack_codes(codes.reshape(-1), 4),
            "scale": scale16, "zero": z.astype(np.float16), "group": group, "shape": (N, K)}


def dequant_int4_group(q: Dict[str, np.ndarray], zero=None) -> np.ndarray:
    N, K = q["shape"]
    L = q["group"]
    z = (q["zero"] if zero is None else zero).astype(np.float32)
    sc = q["scale"].astype(np.float32)
    c = q["codes"].reshape(N, K // L, L).astype(np.float32)
    d = (c - z[..., None]).astype(np.float32)
    v = (d * sc[..., None]).astype(np.float32)
    return bf16_rn(v.reshape(-1)).reshape(N, K)


def qalora_merged_zero_fp64(q: Dict[str, np.ndarray], A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """Unrounded merged zero points z - s (B A) / (L scale) in fp64 (z where scale == 0)."""
    L = q["group"]
    BA = np.asarray(B, np.float64) @ np.asarray(A, np.float64)           # [N, K/L]
    sc = q["scale"].astype(np.float64)
    z = q["zero"].astype(np.float64)
    t = np.float64(np.float32(s)) * BA
    den = np.float64(L) * sc
    with np.errstate(divide="ignore", invalid="ignore"):
        zp = z - t / den
    return np.where(sc > 0, zp, z)


def qalora_merge(q: Dict[str, np.ndarray], A: np.ndarray, B: np.ndarray, s: float) -> np.ndarray:
    """Merged fp16 zero points (fp64 arithmetic, one rounding to fp16)."""
    return qalora_merged_zero_fp64(q, A, B, s).astype(np.float16)
