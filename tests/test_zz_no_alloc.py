"""The no-allocation variant of the adapter-gradient call, for callers that cannot allocate device
memory (a framework owning all device memory, a fixed memory plan, or a loop that must not pay
cudaMalloc/cudaFree).  It must give the results of qlr_backward_lora, call after call, while using
the scratch array built into the library instead of a caller workspace.

This file is named to be collected last, so a run that stops at the first failure has run every
other test first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from synth import LinearSpec, linear_tensors

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


CASES = {
    "nf4": (LinearSpec("w", 1536, 1024, "nfk", 4, 64, 256, r=32, s=0.5), 1024),
    "int4_pooled": (LinearSpec("w", 1024, 2048, "int4g", group=32, r=16, s=1.0, pooled=True), 1024),
    # a problem whose split partial sums fill 13.75 MiB of the 16 MiB array
    "near_limit": (LinearSpec("w", 16384, 1024, "nfk", 4, 64, 256, r=64, s=0.25), 5120),
}


@pytest.mark.parametrize("case", list(CASES))
def test_noalloc_matches_workspace_call_twice(case):
    from quantized_base_lora_nf4_b200 import qlr
    L = qlr.lib()
    dev = "cuda:0"
    spec, M = CASES[case]
    pooled = spec.pooled
    t = linear_tensors(spec, M, seed=3)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16).contiguous()  # noqa
    W = torch.from_numpy(t["W"]).to(dev)
    q = qlr.quantize_int4_group(W, spec.group) if spec.fmt == "int4g" else qlr.quantize_nf4(W, 4, 64, 256)
    X, A, B, dY = bf(t["X"]), bf(t["A"]), bf(t["B"]), bf(t["dY"])
    _, T = qlr.forward(q, X, A, B, spec.s, pooled=pooled)
    # reference: the workspace entry point
    dA_ref, dB_ref, dT_ref = qlr.backward_lora(q, X, dY, T, B, spec.s, pooled=pooled)
    torch.cuda.synchronize()
    qs = q.struct()
    need = L.qlr_backward_lora_workspace_bytes(ctypes.byref(qs), M, spec.r, int(pooled))
    assert 0 < need <= (16 << 20)  # it does use scratch, within the array
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        dA = torch.full_like(dA_ref, float("nan"))
        dB = torch.full_like(dB_ref, float("nan"))
        dT = torch.zeros_like(dT_ref)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        rc = L.qlr_backward_lora_noalloc(ctypes.byref(qs), _ptr(X), _ptr(dY), _ptr(T), _ptr(B), M, spec.r,
                                         float(spec.s), int(pooled), _ptr(dA), _ptr(dB), _ptr(dT), _ptr(status),
                                         stream)
        torch.cuda.synchronize()
        assert rc == 0, (call, rc)
        assert int(status.item()) == 0
        # the same deterministic kernels in the same fixed summation order: identical bits
        for got, ref, what in ((dA, dA_ref, "dA"), (dB, dB_ref, "dB"), (dT, dT_ref, "dT")):
            assert torch.equal(got.view(torch.int32) if got.dtype == torch.float32 else got.view(torch.int16),
                               ref.view(torch.int32) if ref.dtype == torch.float32 else ref.view(torch.int16)), \
                (case, call, what)


def test_noalloc_rejects_problems_beyond_the_scratch():
    from quantized_base_lora_nf4_b200 import qlr
    L = qlr.lib()
    q = qlr.CQWeight()
    q.fmt, q.bits, q.block, q.dq_block, q.group, q.N, q.K = 1, 4, 64, 256, 32, 1 << 16, 1 << 16
    q.codes = q.c1_fp8 = q.s2 = 0x1000
    need = L.qlr_backward_lora_workspace_bytes(ctypes.byref(q), 1 << 16, 64, 0)
    assert need > (16 << 20)
    P = ctypes.c_void_p(0x1000)
    rc = L.qlr_backward_lora_noalloc(ctypes.byref(q), P, P, P, P, 1 << 16, 64, 1.0, 0, P, P, P, None, None)
    assert rc == -8
