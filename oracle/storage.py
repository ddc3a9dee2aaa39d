"""Storage accounting of the quantised formats (oracle; test infrastructure).

QLoRA explainer, "Innovation 2: Double Quantization": one 32-bit constant per
64 weights costs 32/64 = 0.5 bits per weight; quantising the constants to 8 bits
in groups of 256 with one 32-bit constant per group costs 8/64 + 32/(64*256).
"""
from __future__ import annotations


def nf_constant_bits_per_param(block: int, dq_block: int = 0, c1_bits: int = 8, s2_bits: int = 32,
                               fp32_bits: int = 32) -> float:
    if dq_block:
        return c1_bits / block + s2_bits / (block * dq_block)
    return fp32_bits / block


def nf_bits_per_param(bits: int, block: int, dq_block: int = 0) -> float:
    return bits + nf_constant_bits_per_param(block, dq_block)


def int4g_bits_per_param(group: int) -> float:
    return 4 + (16 + 16) / group


def nf_bytes(N: int, K: int, bits: int, block: int, dq_block: int = 0) -> dict:
    n = N * K
    nb = -(-n // block)
    padded = nb * block
    out = {"codes": padded * bits // 8}
    if dq_block:
        out["c1_fp8"] = nb
        out["s2"] = 4 * (-(-nb // dq_block))
    else:
        out["c1"] = 4 * nb
    return out


def int4g_bytes(N: int, K: int, group: int) -> dict:
    return {"codes": N * K // 2, "scale": 2 * N * (K // group), "zero": 2 * N * (K // group)}
