"""CPU tests of the C-ABI library: it loads without a GPU, exports every symbol include/qlr.h
declares, rejects invalid calls on the host before launching anything, and derives the same
fp32 NF-k tables as the oracle from its own inverse normal."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle.codebook import nf_codebook_f32
from oracle import storage

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from quantized_base_lora_nf4_b200 import build, qlr
    build.build()
    return qlr.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "qlr.h")).read()
    return sorted(set(re.findall(r"QLR_API\s+[\w\s\*]+?\b(qlr_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = declared_symbols()
    for required in ("qlr_quantize_nf4", "qlr_quantize_int4_group", "qlr_forward", "qlr_backward_dx",
                     "qlr_backward_lora", "qlr_qalora_merge", "qlr_dequant"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_binding_covers_header(L):
    from quantized_base_lora_nf4_b200 import qlr
    assert set(qlr.EXPORTED) <= set(declared_symbols())


def test_error_strings(L):
    for code in range(-8, 1):
        assert L.qlr_error_string(code)
    assert L.qlr_version() >= 100


@pytest.mark.parametrize("k", [2, 3, 4])
def test_library_levels_match_oracle_bit_for_bit(L, k):
    from quantized_base_lora_nf4_b200 import qlr
    lv = qlr.nf_levels(k).numpy()
    np.testing.assert_array_equal(lv.view(np.uint32), nf_codebook_f32(k).view(np.uint32))


def test_part_bytes_match_storage_accounting(L):
    from quantized_base_lora_nf4_b200 import qlr
    for (N, K, b, blk, dq) in [(28672, 8192, 4, 64, 256), (4096, 11008, 3, 128, 256), (256, 256, 2, 64, 0)]:
        ref = storage.nf_bytes(N, K, b, blk, dq)
        assert qlr.part_bytes(qlr.FMT_NFK, N, K, b, blk, dq, 32, qlr.PART_CODES) == ref["codes"]
        if dq:
            assert qlr.part_bytes(qlr.FMT_NFK, N, K, b, blk, dq, 32, qlr.PART_C1_FP8) == ref["c1_fp8"]
            assert qlr.part_bytes(qlr.FMT_NFK, N, K, b, blk, dq, 32, qlr.PART_S2) == ref["s2"]
        else:
            assert qlr.part_bytes(qlr.FMT_NFK, N, K, b, blk, dq, 32, qlr.PART_C1) == ref["c1"]
    g = storage.int4g_bytes(4096, 4096, 32)
    assert qlr.part_bytes(qlr.FMT_INT4G, 4096, 4096, 4, 64, 0, 32, qlr.PART_SCALE) == g["scale"]
    assert qlr.part_bytes(qlr.FMT_INT4G, 4096, 4096, 4, 64, 0, 32, qlr.PART_CODES) == g["codes"]
    with pytest.raises(qlr.QLRError):
        qlr.part_bytes(qlr.FMT_NFK, 16, 64, 5, 64, 256, 32, qlr.PART_CODES)


def _fake_qweight(fmt=1, bits=4, block=64, dq=256, group=32, N=256, K=256, ptr=0x1000):
    from quantized_base_lora_nf4_b200.qlr import CQWeight
    q = CQWeight()
    q.fmt, q.bits, q.block, q.dq_block, q.group, q.N, q.K = fmt, bits, block, dq, group, N, K
    q.codes = q.c1 = q.c1_fp8 = q.s2 = q.scale = q.zero = ptr
    return q


def test_host_validation_rejects_before_launch(L):
    """Every call below fails in argument checking; none reaches the CUDA runtime."""
    q = _fake_qweight()
    P = ctypes.c_void_p
    # null weight / input
    assert L.qlr_quantize_nf4(None, 256, 256, 4, 64, 256, ctypes.byref(q), None, None) == -1
    # metadata mismatch
    assert L.qlr_quantize_nf4(P(0x1000), 256, 256, 4, 128, 256, ctypes.byref(q), None, None) == -1
    # misaligned input pointer
    assert L.qlr_quantize_nf4(P(0x1004), 256, 256, 4, 64, 256, ctypes.byref(q), None, None) == -3
    # bad block / bits
    bad = _fake_qweight(block=96)
    assert L.qlr_quantize_nf4(P(0x1000), 256, 256, 4, 96, 256, ctypes.byref(bad), None, None) == -1
    # rank not supported
    assert L.qlr_forward(ctypes.byref(q), P(0x1000), 16, P(0x1000), P(0x1000), 12, 1.0, 0, P(0x1000), P(0x1000),
                         P(0x1000), 1 << 20, None, None) == -2
    # K not a multiple of 64 for the tensor-core paths
    q2 = _fake_qweight(K=96 * 4, N=8)
    q2.K = 200
    assert L.qlr_forward(ctypes.byref(q2), P(0x1000), 16, P(0x1000), P(0x1000), 8, 1.0, 0, P(0x1000), P(0x1000),
                         P(0x1000), 1 << 20, None, None) in (-2,)
    # pooled adapter with an NF weight
    assert L.qlr_forward(ctypes.byref(q), P(0x1000), 16, P(0x1000), P(0x1000), 8, 1.0, 1, P(0x1000), P(0x1000),
                         P(0x1000), 1 << 20, None, None) == -4
    # 3-bit codes stream two 64-code steps per box along K: K must be a multiple of 128
    q3 = _fake_qweight(bits=3, K=192)
    assert L.qlr_forward(ctypes.byref(q3), P(0x1000), 16, P(0x1000), P(0x1000), 8, 1.0, 0, P(0x1000), P(0x1000),
                         P(0x1000), 1 << 20, None, None) == -2
    # missing workspace (64 tokens: the adapter GEMM's split partial sums need one)
    assert L.qlr_forward(ctypes.byref(q), P(0x1000), 64, P(0x1000), P(0x1000), 8, 1.0, 0, P(0x1000), P(0x1000),
                         None, 0, None, None) == -8
    # merge needs an INT4 group weight
    assert L.qlr_qalora_merge(ctypes.byref(q), P(0x1000), P(0x1000), 8, 1.0, None, None) == -1
    # swiglu element count must be a multiple of 8
    assert L.qlr_swiglu_forward(P(0x1000), P(0x1000), P(0x1000), 12, None) == -2
    assert L.qlr_swiglu_forward(P(0x1000), P(0x1000), P(0x1000), -1, None) == -1
