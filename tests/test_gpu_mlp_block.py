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


def run_block(qlr, specs, M, seed, rows=None):
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
    U = qlr.forward_base(qs[1], Xd, B[1], Tu, status=st)
    H = qlr.swiglu_forward(G, U)
    Td = qlr.lora_down(qs[2], H, A[2], ds.s, status=st)
    Y = qlr.forward_base(qs[2], H, B[2], Td, status=st)
    # backward
    dAd, dBd, dTd = qlr.backward_lora(qs[2], H, dOutd, Td, B[2], ds.s, status=st)
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
    check_close(host(dH)[sel], bd["dX"][sel], "dH")
    check_close(host(dG)[sel], dg[sel], "dG")
    check_close(host(dU)[sel], du[sel], "dU")
    check_close(host(dX)[sel], (bg["dX"] + bu["dX"])[sel], "dX = gate's + up's")
    for got, ref, what in ((dAd, bd["dA"], "dA down"), (dBd, bd["dB"], "dB down"), (dAg, bg["dA"], "dA gate"),
                           (dBg, bg["dB"], "dB gate"), (dAu, bu["dA"], "dA up"), (dBu, bu["dB"], "dB up")):
        check_close(host(got), ref, what)


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
