"""Pins for the storage accounting against the figures the pages print (tests/golden/page_figures.json)."""
import json
import os

import pytest

from oracle import storage
from oracle.codebook import nf_codebook

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def v(name):
    return GOLD[name]["value"]


def test_constant_overheads():
    assert storage.nf_constant_bits_per_param(64) == v("constant_bits_fp32_block64")
    dq = storage.nf_constant_bits_per_param(64, 256)
    assert dq == pytest.approx(8 / 64 + 32 / (64 * 256), abs=0)
    assert round(dq, 3) == v("constant_bits_double_quant")
    saving = storage.nf_constant_bits_per_param(64) - dq
    assert round(saving, 2) == v("double_quant_saving_bits")


def test_65b_figures():
    n = 65e9
    assert round(n * storage.nf_constant_bits_per_param(64) / 8 / 1e9) == v("constants_65b_gb")
    saving = n * (storage.nf_constant_bits_per_param(64) - storage.nf_constant_bits_per_param(64, 256)) / 8 / 1e9
    assert round(saving) == v("double_quant_saving_65b_gb")
    assert n * 16 / 8 / 1e9 == v("weights_65b_16bit_gb")
    shrink = 16 / storage.nf_bits_per_param(4, 64, 256)
    assert abs(shrink - v("nf4_shrink_vs_16bit")) / v("nf4_shrink_vs_16bit") < 0.05


def test_nf4_level_count():
    assert nf_codebook(4).size == v("nf4_levels")


def test_lqlora_budget_arithmetic():
    gb = 70e9 * v("lqlora_70b_avg_bits_with_lowrank") / 8 / 1e9
    assert gb <= v("lqlora_70b_gb")


def test_byte_counts():
    b = storage.nf_bytes(28672, 8192, 4, 64, 256)
    assert b["codes"] == 28672 * 8192 // 2
    assert b["c1_fp8"] == 28672 * 8192 // 64
    assert b["s2"] == 4 * (28672 * 8192 // 64 // 256)
    g = storage.int4g_bytes(4096, 4096, 32)
    assert g == {"codes": 4096 * 2048, "scale": 2 * 4096 * 128, "zero": 2 * 4096 * 128}
    assert storage.int4g_bits_per_param(32) == 5.0
