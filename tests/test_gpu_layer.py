"""GPU parity of the forward / backward entry points against the fp64 oracle
(relative Frobenius error <= 1e-2, the bound stated for the bf16 paths)."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import quantize as Q
from synth import LinearSpec, linear_tensors, workload, random_matrix
from tests.gpu_helpers import DEV, bf16_dev, f32_dev, host

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]

TOL = 1e-2
# a single token row (or weight row) may be off by at most this much relative to its own norm: the
# whole-tensor bound alone would let one row of 2048 be 45 % wrong
ROW_TOL = 3e-2


def worst_row(got, ref, axis=1):
    """Largest error of one row (axis=1) or column (axis=0), relative to that row's norm, the norm floored
    at a tenth of the mean so that a row whose exact value nearly cancels is not judged on its own."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    num = np.linalg.norm(got - ref, axis=axis)
    den = np.linalg.norm(ref, axis=axis)
    den = np.maximum(den, 0.1 * den.mean() + 1e-300)
    return float((num / den).max())


def check_close(got, ref, what):
    """The relative Frobenius bound on the whole tensor, and the per-row (and, with 8 or more rows,
    per-column) bound, so an error confined to one token, one weight row, one tile or a ragged tail shows."""
    got = np.asarray(got, np.float64)
    assert OL.rel_fro(got, ref) <= TOL, (what, OL.rel_fro(got, ref))
    if got.ndim == 2 and got.size:
        assert worst_row(got, ref, 1) <= ROW_TOL, (what, "row", worst_row(got, ref, 1))
        if got.shape[0] >= 8:
            assert worst_row(got, ref, 0) <= ROW_TOL, (what, "column", worst_row(got, ref, 0))


def quantize_both(qlr, spec, W):
    if spec.fmt == "int4g":
        ref = Q.quantize_int4_group(W, spec.group)
        return qlr.quantize_int4_group(f32_dev(W), spec.group), Q.dequant_int4_group(ref)
    ref = Q.quantize_nfk(W, spec.bits, spec.block, spec.dq_block)
    return qlr.quantize_nf4(f32_dev(W), spec.bits, spec.block, spec.dq_block), Q.dequant_nfk(ref)


def run_and_check(qlr, spec, M, seed=0, rows=None, accumulate_check=False):
    t = linear_tensors(spec, M, seed=seed)
    q, Wdq = quantize_both(qlr, spec, t["W"])
    X, A, B, dY = bf16_dev(t["X"]), bf16_dev(t["A"]), bf16_dev(t["B"]), bf16_dev(t["dY"])
    st = qlr.new_status(DEV)
    Y, T = qlr.forward(q, X, A, B, spec.s, pooled=spec.pooled, status=st)
    dA, dB, dT = qlr.backward_lora(q, X, dY, T, B, spec.s, pooled=spec.pooled, status=st)
    dX = qlr.backward_dx(q, dY, A, dT, pooled=spec.pooled, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    L = spec.group if spec.pooled else None
    sel = slice(None) if rows is None else rows
    Xs, dYs = t["X"][sel], t["dY"][sel]
    f = OL.forward(Xs, Wdq, t["A"], t["B"], spec.s, L)
    check_close(host(Y)[sel], f["Y"], "Y")
    check_close(host(T)[sel], spec.s * f["T"], "T")
    bsel = OL.backward(dYs, Xs, Wdq, t["A"], t["B"], spec.s, L)
    check_close(host(dT)[sel], bsel["dT"], "dT")
    check_close(host(dX)[sel], bsel["dX"], "dX")
    # adapter gradients reduce over every token: checked in full
    full = bsel if rows is None else OL.backward(t["dY"], t["X"], Wdq, t["A"], t["B"], spec.s, L)
    check_close(host(dA), full["dA"], "dA")
    check_close(host(dB), full["dB"], "dB")
    if accumulate_check:
        dX2 = dX.clone()
        qlr.backward_dx(q, dY, A, dT, pooled=spec.pooled, dX=dX2, accumulate=True)
        torch.cuda.synchronize()
        check_close(host(dX2)[sel], 2 * bsel["dX"], "dX accumulated")
    return {"Y": Y, "dX": dX, "dA": dA, "dB": dB}


def test_tiny_layer(cuda_lib):
    wl = workload("tiny")
    run_and_check(cuda_lib, wl.linears[0], wl.M, accumulate_check=True)


@pytest.mark.parametrize("M", [1, 40, 200, 333, 700])
@pytest.mark.parametrize("r", [8, 16, 32, 64])
def test_ragged_nf4(cuda_lib, M, r):
    spec = LinearSpec("w", 320, 384, "nfk", 4, 128, 0, r=r, s=0.5)
    run_and_check(cuda_lib, spec, M, seed=M + r)


@pytest.mark.parametrize("bits", [2, 3])
@pytest.mark.parametrize("M,r,block,dq", [(1, 8, 64, 256), (40, 64, 128, 0), (333, 16, 64, 256), (700, 32, 128, 256)])
def test_ragged_nf_low_bits(cuda_lib, bits, M, r, block, dq):
    """NF-2 and NF-3 codes (LQ-LoRA's per-matrix bit widths) through the fused forward and input
    gradient: 2-bit codes in 16-byte runs, 3-bit bit planes two steps per codes box."""
    spec = LinearSpec("w", 320, 384, "nfk", bits, block, dq, r=r, s=0.5)
    run_and_check(cuda_lib, spec, M, seed=100 * bits + M)


@pytest.mark.parametrize("bits", [2, 3])
def test_lqlora_matrix_full_size_sampled_rows(cuda_lib, bits):
    """The first matrix of the mixed 7B stack drawn with this bit width, at its full shape and 2048 tokens."""
    wl = workload("lqlora")
    idx = next(i for i, s in enumerate(wl.linears) if s.bits == bits)
    spec = wl.linears[idx]
    rows = np.sort(np.random.default_rng(bits).choice(wl.M, 96, replace=False))
    run_and_check(cuda_lib, spec, wl.M, seed=idx, rows=rows)


@pytest.mark.parametrize("M", [64, 300, 1100])
def test_ragged_int4_pooled(cuda_lib, M):
    spec = LinearSpec("w", 264, 512, "int4g", group=32, r=16, s=1.0, pooled=True)
    run_and_check(cuda_lib, spec, M, seed=7)


def test_int4_unpooled_and_group64(cuda_lib):
    run_and_check(cuda_lib, LinearSpec("w", 256, 512, "int4g", group=64, r=8, s=2.0, pooled=False), 96, seed=9)


def test_qalora_full_size(cuda_lib):
    wl = workload("qalora")
    run_and_check(cuda_lib, wl.linears[0], wl.M)


@pytest.mark.parametrize("which", [0, 2])
def test_mlp7b_full_size_sampled_rows(cuda_lib, which):
    wl = workload("mlp7b")
    spec = wl.linears[which]
    rows = np.sort(np.random.default_rng(which).choice(wl.M, 128, replace=False))
    run_and_check(cuda_lib, spec, wl.M, rows=rows)


def test_swiglu(cuda_lib):
    qlr = cuda_lib
    G = random_matrix(31, 0, "X", (64, 1024), 2.0, bf16=True)
    U = random_matrix(31, 1, "X", (64, 1024), 1.0, bf16=True)
    dH = random_matrix(31, 2, "X", (64, 1024), 1.0, bf16=True)
    H = qlr.swiglu_forward(bf16_dev(G), bf16_dev(U))
    dG, dU = qlr.swiglu_backward(bf16_dev(dH), bf16_dev(G), bf16_dev(U))
    torch.cuda.synchronize()
    check_close(host(H), OL.swiglu_forward(G, U), "H")
    rg, ru = OL.swiglu_backward(dH, G, U)
    check_close(host(dG), rg, "dG")
    check_close(host(dU), ru, "dU")


def test_zero_tokens(cuda_lib):
    qlr = cuda_lib
    spec = LinearSpec("w", 128, 256, "nfk", 4, 64, 256, r=8, s=1.0)
    t = linear_tensors(spec, 4, seed=1)
    q, _ = quantize_both(qlr, spec, t["W"])
    X = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    dY = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    Y, T = qlr.forward(q, X, bf16_dev(t["A"]), bf16_dev(t["B"]), 1.0)
    dA, dB, dT = qlr.backward_lora(q, X, dY, T, bf16_dev(t["B"]), 1.0)
    torch.cuda.synchronize()
    assert Y.shape == (0, 128) and float(dA.abs().sum()) == 0 and float(dB.abs().sum()) == 0


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_projection_full_size_sampled_rows(cuda_lib, M):
    """The 28672 x 8192 NF4+DQ projection at decode token counts (the HBM-bound decode kernel):
    output features checked on whole double-quantisation groups of sampled weight rows."""
    qlr = cuda_lib
    wl = workload("decode70b")
    spec = wl.linears[0]
    t = linear_tensors(spec, 16, seed=0, with_dy=False)
    q = qlr.quantize_nf4(f32_dev(t["W"]), 4, 64, 256)
    X = t["X"][:M]
    Y, T = qlr.forward(q, bf16_dev(X), bf16_dev(t["A"]), bf16_dev(t["B"]), spec.s)
    torch.cuda.synchronize()
    Yh = host(Y)
    rows = np.sort(np.random.default_rng(M).choice(spec.N // 2, 48, replace=False)) * 2
    sel = np.concatenate([[r, r + 1] for r in rows])
    Wdq = np.concatenate([Q.dequant_nfk(Q.quantize_nfk(t["W"][r:r + 2], 4, 64, 256)) for r in rows])
    ref = OL.forward(X, np.zeros((2 * len(rows), spec.K)), t["A"], t["B"][sel], spec.s)["Y"] + \
        X.astype(np.float64) @ Wdq.astype(np.float64).T
    check_close(Yh[:, sel], ref, "Y")
    check_close(host(T), spec.s * OL.forward(X, np.zeros((1, spec.K)), t["A"], t["B"][:1], spec.s)["T"], "T")


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("block,r", [(64, 8), (128, 64)])
def test_decode_ragged(cuda_lib, M, block, r):
    """Decode kernel (256-input steps) on a weight whose 20 units of 16 rows give one unit per CTA and whose
    rows do not fill the last unit: 312 rows, K = 768 (three steps, an odd count)."""
    spec = LinearSpec("w", 312, 768, "nfk", 4, block, 256, r=r, s=0.5)
    run_and_check(cuda_lib, spec, M, seed=11 + M)


def test_several_tiles_per_cta_without_token_pairs(cuda_lib):
    # 10240 rows (and 10240 reduction columns for dX) give 80 row tiles; 100 tokens take two 64-token
    # tiles and 300 tokens two 256-token tiles, so 160 tiles run on at most 148 persistent CTAs and some
    # CTAs alternate their two TMEM accumulators across tiles, in the forward and in the input gradient
    qlr = cuda_lib
    spec = LinearSpec("w", 10240, 10240, "nfk", 4, 64, 256, r=16, s=0.5)
    t0 = linear_tensors(spec, 300, seed=31)
    q, Wdq = quantize_both(qlr, spec, t0["W"])
    for M in (100, 300):
        X, dY = t0["X"][:M], t0["dY"][:M]
        st = qlr.new_status(DEV)
        A, B = bf16_dev(t0["A"]), bf16_dev(t0["B"])
        Y, T = qlr.forward(q, bf16_dev(X), A, B, spec.s, status=st)
        dA, dB, dT = qlr.backward_lora(q, bf16_dev(X), bf16_dev(dY), T, B, spec.s, status=st)
        dX = qlr.backward_dx(q, bf16_dev(dY), A, dT, status=st)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        f = OL.forward(X, Wdq, t0["A"], t0["B"], spec.s)
        b = OL.backward(dY, X, Wdq, t0["A"], t0["B"], spec.s)
        check_close(host(Y), f["Y"], "Y")
        check_close(host(dX), b["dX"], "dX")
        check_close(host(dA), b["dA"], "dA")
        check_close(host(dB), b["dB"], "dB")


@pytest.mark.parametrize("pooled", [False, True])
def test_split_adapter_backward_on_two_streams_bit_identical(cuda_lib, pooled):
    """dT on one stream, then dB and dA on a second stream that waits for it (beside the input gradient on the
    first): the same kernels as backward_lora in one call, so the same bits."""
    qlr = cuda_lib
    if pooled:
        spec = LinearSpec("w", 1024, 2048, "int4g", group=32, r=16, s=1.0, pooled=True)
    else:
        spec = LinearSpec("w", 1536, 1024, "nfk", 3, 128, 256, r=64, s=0.25)
    M = 700
    t = linear_tensors(spec, M, seed=12)
    q, _ = quantize_both(qlr, spec, t["W"])
    X, A, B, dY = bf16_dev(t["X"]), bf16_dev(t["A"]), bf16_dev(t["B"]), bf16_dev(t["dY"])
    _, T = qlr.forward(q, X, A, B, spec.s, pooled=pooled)
    dA0, dB0, dT0 = qlr.backward_lora(q, X, dY, T, B, spec.s, pooled=pooled)
    dX0 = qlr.backward_dx(q, dY, A, dT0, pooled=pooled)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    st = qlr.new_status(DEV)
    dT = qlr.backward_lora_dT(q, dY, B, spec.s, status=st)
    ev = torch.cuda.Event()
    ev.record(main)
    side.wait_event(ev)
    dA, dB = qlr.backward_lora_dAdB(q, X, dY, T, dT, pooled=pooled, status=st, stream=side)
    dX = qlr.backward_dx(q, dY, A, dT, pooled=pooled, status=st)
    main.wait_stream(side)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for a, b in ((dT, dT0), (dX, dX0)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for a, b in ((dA, dA0), (dB, dB0)):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("N,K", [(11008, 512), (512, 11008)])
def test_last_wave_split_into_half_tiles(cuda_lib, N, K):
    """2048 tokens over 86 row tiles give 344 tiles of 128 x 512 on 148 SMs: the 48 tiles of the last wave
    are split into 96 half tiles of 256 tokens (forward for N = 11008, input gradient for K = 11008)."""
    spec = LinearSpec("w", N, K, "nfk", 4, 64, 256, r=16, s=0.5)
    rows = np.sort(np.random.default_rng(N).choice(2048, 160, replace=False))
    run_and_check(cuda_lib, spec, 2048, seed=17, rows=rows)
