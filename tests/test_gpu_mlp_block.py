"""GPU parity of the chained MLP block (gate/up -> SwiGLU -> down, forward and backward) against the fp64
oracle, run the way the training step runs it: the up projection's input gradient accumulates onto the
gate's, and every intermediate (G, U, H, dH, dG, dU) stays in bf16 on the device between the calls.

The block is the LLaMA-7B-shaped MLP workload (gate/up 11008 x 4096, down 4096 x 11008, NF4 with double
quantisation, r = 64, s = 16/64) and a reduced copy of it with a ragged token count."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from synth import LinearSpec, linear_tensors, workload
from tests.gpu_helpers import DEV, bf16_dev, host
from tests.test_gpu_layer import check_close, quantize_both

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]


def run_block(qlr, specs, M, seed, rows=None, fused=False):
    """The block on the GPU (fused: SwiGLU inside the up projection's and the down projection's input-gradient
    epilogues) checked against the oracle's chain; returns every device result."""
    gs, us, ds = specs
    ts = [linear_tensors(s, M, seed=seed, matrix_index=i, with_x=(i == 0), with_dy=(i == 2)) for i, s in enumerate(specs)]
    X = ts[0]["X"]
    dOut = ts[2]["dY"]
    qs, Wdq = zip(*[quantize_both(qlr, s, t["W"]) for s, t in zip(specs, ts)])
    A = [bf16_dev(t["A"]) for t in ts]
    B = [bf16_dev(t["B"]) for t in ts]
    st = qlr.new_status(DEV)
    Xd, dOutd = bf16_dev(X), bf16_dev(dOut)
    # forward
    Tg = qlr.lora_down(qs[0], Xd, A[0], gs.s, status=st)
    Tu = qlr.lora_down(qs[1], Xd, A[1], us.s, status=st)
    G = qlr.forward_base(qs[0], Xd, B[0], Tg, status=st)
    if fused:
        U, H = qlr.forward_swiglu(qs[1], Xd, B[1], Tu, G, status=st)
    else:
        U = qlr.forward_base(qs[1], Xd, B[1], Tu, status=st)
        H = qlr.swiglu_forward(G, U)
    Td = qlr.lora_down(qs[2], H, A[2], ds.s, status=st)
    Y = qlr.forward_base(qs[2], H, B[2], Td, status=st)
    # backward
    dAd, dBd, dTd = qlr.backward_lora(qs[2], H, dOutd, Td, B[2], ds.s, status=st)
    if fused:
        dH = None
        dG, dU = qlr.backward_dx_swiglu(qs[2], dOutd, A[2], dTd, G, U, status=st)
    else:
        dH = qlr.backward_dx(qs[2], dOutd, A[2], dTd, status=st)
        dG, dU = qlr.swiglu_backward(dH, G, U)
    dAg, dBg, dTg = qlr.backward_lora(qs[0], Xd, dG, Tg, B[0], gs.s, status=st)
    dX = qlr.backward_dx(qs[0], dG, A[0], dTg, status=st)
    dAu, dBu, dTu = qlr.backward_lora(qs[1], Xd, dU, Tu, B[1], us.s, status=st)
    qlr.backward_dx(qs[1], dU, A[1], dTu, dX=dX, accumulate=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0

    # the oracle's chain, fp64 from the same inputs
    g = OL.forward(X, Wdq[0], ts[0]["A"], ts[0]["B"], gs.s)["Y"]
    u = OL.forward(X, Wdq[1], ts[1]["A"], ts[1]["B"], us.s)["Y"]
    h = OL.swiglu_forward(g, u)
    bd = OL.backward(dOut, h, Wdq[2], ts[2]["A"], ts[2]["B"], ds.s)
    dg, du = OL.swiglu_backward(bd["dX"], g, u)
    bg = OL.backward(dg, X, Wdq[0], ts[0]["A"], ts[0]["B"], gs.s)
    bu = OL.backward(du, X, Wdq[1], ts[1]["A"], ts[1]["B"], us.s)
    sel = slice(None) if rows is None else rows
    y = OL.forward(h[sel], Wdq[2], ts[2]["A"], ts[2]["B"], ds.s)["Y"]
    check_close(host(Y)[sel], y, "Y")
    check_close(host(H)[sel], h[sel], "H")
    if dH is not None:
        check_close(host(dH)[sel], bd["dX"][sel], "dH")
    check_close(host(dG)[sel], dg[sel], "dG")
    check_close(host(dU)[sel], du[sel], "dU")
    check_close(host(dX)[sel], (bg["dX"] + bu["dX"])[sel], "dX = gate's + up's")
    for got, ref, what in ((dAd, bd["dA"], "dA down"), (dBd, bd["dB"], "dB down"), (dAg, bg["dA"], "dA gate"),
                           (dBg, bg["dB"], "dB gate"), (dAu, bu["dA"], "dA up"), (dBu, bu["dB"], "dB up")):
        check_close(host(got), ref, what)
    return {"Y": Y, "G": G, "U": U, "H": H, "dG": dG, "dU": dU, "dX": dX, "dAd": dAd, "dBd": dBd, "dAg": dAg,
            "dBg": dBg, "dAu": dAu, "dBu": dBu}


def test_mlp_block_reduced_ragged(cuda_lib):
    """Hidden 512, intermediate 704 (11 steps of 64), 300 tokens: several tiles and a ragged tail everywhere."""
    s = 16.0 / 64.0
    specs = (LinearSpec("gate", 704, 512, "nfk", 4, 64, 256, r=16, s=s),
             LinearSpec("up", 704, 512, "nfk", 4, 64, 256, r=16, s=s),
             LinearSpec("down", 512, 704, "nfk", 4, 64, 256, r=16, s=s))
    run_block(cuda_lib, specs, 300, seed=41)


def test_mlp_block_full_size_sampled_rows(cuda_lib):
    """The LLaMA-7B MLP block at 4096 tokens: token rows of Y, H, dH, dG, dU and dX on 96 sampled rows
    (rows are independent through the block), the six adapter gradients in full."""
    wl = workload("mlp7b")
    rows = np.sort(np.random.default_rng(5).choice(wl.M, 96, replace=False))
    run_block(cuda_lib, wl.linears, wl.M, seed=0, rows=rows)


@pytest.mark.parametrize("M", [300, 8])
def test_mlp_block_swiglu_fused_bit_identical(cuda_lib, M):
    """The SwiGLU fused into the up projection's epilogue (forward) and the down projection's input-gradient
    epilogue (backward) gives exactly the bits of the separate SwiGLU kernels (one shared definition of the
    arithmetic), and matches the oracle.  8 tokens: the up projection runs the decode kernel, then SwiGLU."""
    s = 16.0 / 64.0
    # the decode kernel (8 tokens) needs K a multiple of 256: gate/up K = 512, down K = 768
    specs = (LinearSpec("gate", 768, 512, "nfk", 4, 64, 256, r=16, s=s),
             LinearSpec("up", 768, 512, "nfk", 4, 64, 256, r=16, s=s),
             LinearSpec("down", 512, 768, "nfk", 4, 64, 256, r=16, s=s))
    a = run_block(cuda_lib, specs, M, seed=43)
    b = run_block(cuda_lib, specs, M, seed=43, fused=True)
    for k, v in a.items():
        assert torch.equal(v.view(torch.int16) if v.dtype == torch.bfloat16 else v.view(torch.int32),
                           b[k].view(torch.int16) if b[k].dtype == torch.bfloat16 else b[k].view(torch.int32)), k


def test_mlp_block_full_size_fused(cuda_lib):
    wl = workload("mlp7b")
    rows = np.sort(np.random.default_rng(6).choice(wl.M, 64, replace=False))
    run_block(cuda_lib, wl.linears, wl.M, seed=0, rows=rows, fused=True)
