"""Failure detection without a fault: the pipelined kernels' bounded waits.

Every handshake of the fused GEMM, the adapter GEMM and the decode kernel waits for at most a bound of SM
clock cycles; past it the kernel raises an abort flag, drains its own copies and tensor-core work in flight,
releases its tensor memory and reports QLR_ERR_TIMEOUT in the status word.  These tests make the waits run
out without faulting anything: a self-test kernel waits on a barrier nothing completes, and the real
kernels run with a bound of zero cycles (any wait not already complete after 64 polls gives up).  After each
timeout a normal call on the same device must succeed and give the same bits as before, which shows the
context is intact and the tensor memory was released.
"""
import time

import pytest
import torch

from oracle import layer as OL
from oracle import quantize as Q
from synth import linear_tensors, workload
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]

TIMEOUT = -6


@pytest.fixture
def default_limit(cuda_lib):
    yield cuda_lib
    cuda_lib.set_wait_limit(-1)


def test_selftest_wait_times_out_and_releases_tensor_memory(default_limit):
    qlr = default_limit
    qlr.set_wait_limit(2_000_000)  # about a millisecond
    st = qlr.new_status(DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    qlr.wait_selftest(st)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 1.0
    assert int(st.item()) == TIMEOUT
    qlr.set_wait_limit(-1)
    # the tiny layer, forward and backward, right after: its kernels allocate tensor memory again
    spec = workload("tiny").linears[0]
    t = linear_tensors(spec, 16, seed=0)
    q = qlr.quantize_nf4(f32_dev(t["W"]), 4, 64, 256)
    st = qlr.new_status(DEV)
    X, A, B, dY = bf16_dev(t["X"]), bf16_dev(t["A"]), bf16_dev(t["B"]), bf16_dev(t["dY"])
    Y, T = qlr.forward(q, X, A, B, spec.s, status=st)
    dA, dB, dT = qlr.backward_lora(q, X, dY, T, B, spec.s, status=st)
    dX = qlr.backward_dx(q, dY, A, dT, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    Wdq = Q.dequant_nfk(Q.quantize_nfk(t["W"], 4, 64, 256))
    f = OL.forward(t["X"], Wdq, t["A"], t["B"], spec.s)
    b = OL.backward(t["dY"], t["X"], Wdq, t["A"], t["B"], spec.s)
    for got, ref in ((Y, f["Y"]), (dX, b["dX"]), (dA, b["dA"]), (dB, b["dB"])):
        assert OL.rel_fro(host(got), ref) <= 1e-2


def _layer(qlr, N, K, M, r=64, seed=3):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    W = torch.randn((N, K), generator=g, device=DEV) * 0.02
    q = qlr.quantize_nf4(W, 4, 64, 256)
    mk = lambda *s: (torch.randn(s, generator=g, device=DEV)).to(torch.bfloat16)  # noqa: E731
    return q, mk(M, K), (mk(r, K) * 0.01).to(torch.bfloat16), (mk(N, r) * 0.01).to(torch.bfloat16), mk(M, N)


def _bits(ts):
    return [t.view(torch.int16).clone() if t.dtype == torch.bfloat16 else t.view(torch.int32).clone() for t in ts]


@pytest.mark.parametrize("path", ["forward", "backward_dx", "backward_lora", "decode"])
def test_pipeline_kernels_time_out_cleanly(default_limit, path):
    qlr = default_limit
    M = 4 if path == "decode" else 2048
    q, X, A, B, dY = _layer(qlr, 8192, 4096, M)

    def run(st):
        if path in ("forward", "decode"):
            return qlr.forward(q, X, A, B, 0.25, status=st)
        T = qlr.lora_down(q, X, A, 0.25)
        if path == "backward_lora":
            return qlr.backward_lora(q, X, dY, T, B, 0.25, status=st)
        dA, dB, dT = qlr.backward_lora(q, X, dY, T, B, 0.25)
        return (qlr.backward_dx(q, dY, A, dT, status=st),)

    st = qlr.new_status(DEV)
    before = _bits(run(st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    qlr.set_wait_limit(0)
    st = qlr.new_status(DEV)
    t0 = time.perf_counter()
    run(st)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(st.item()) == TIMEOUT
    qlr.set_wait_limit(-1)
    st = qlr.new_status(DEV)
    after = _bits(run(st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for a, b in zip(before, after):
        assert torch.equal(a, b)
