"""LQ-LoRA initialisation on the GPU against the oracle.

The SVD is single precision on the GPU and double in the oracle, so the low-rank parts agree to
rounding and a handful of codes that sit on a level boundary may quantise differently; the tests
compare what is unique (the low-rank product s B A, the reconstruction error, the code agreement)
and require plain quantisation (no iteration) to be bit-exact."""
import numpy as np
import pytest
import torch

from oracle import layer as OL
from oracle import lqlora as LQ
from oracle import quantize as Q
from synth import random_matrix

from gpu_helpers import DEV, f32_dev, host, host_bytes

pytestmark = pytest.mark.gpu


def _codes(packed: np.ndarray, bits: int, count: int) -> np.ndarray:
    return Q.unpack_codes(packed, bits, count)


def _run(qlr, W, bits, block, dq, r, s, iters):
    st = qlr.new_status(DEV)
    q, A, B = qlr.lqlora_init(f32_dev(W), bits, block, dq, r, s, iters, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return q, A, B


def test_zero_iterations_is_bit_exact_quantisation(cuda_lib):
    W = random_matrix(5, 0, "W", (96, 384), 0.02)
    q, A, B = _run(cuda_lib, W, 3, 64, 256, 8, 0.25, 0)
    ref = Q.quantize_nfk(W, 3, 64, 256)
    assert np.array_equal(host_bytes(q.codes)[: ref["packed"].size], ref["packed"])
    assert float(A.float().abs().sum()) == 0 and float(B.float().abs().sum()) == 0


@pytest.mark.parametrize("shape", [(96, 384), (384, 128)])  # K >= N (factors R^T) and N > K (transposed)
@pytest.mark.parametrize("bits,block,dq,r,iters", [(4, 64, 256, 8, 1), (2, 128, 0, 16, 2), (3, 64, 256, 16, 3)])
def test_iterations_match_the_oracle(cuda_lib, shape, bits, block, dq, r, iters):
    N, K = shape
    rng_seed = 10 * bits + iters
    # a strong low-rank component plus noise, as in a pretrained matrix with a dominant subspace
    W = (random_matrix(rng_seed, 0, "A", (N, r), 1.0) @ random_matrix(rng_seed, 0, "B", (r, K), 1.0) * 0.02
         + random_matrix(rng_seed, 0, "W", (N, K), 0.01)).astype(np.float32)
    s = 0.25
    q, A, B = _run(cuda_lib, W, bits, block, dq, r, s, iters)
    ref = LQ.lqlora_init(W, bits, block, dq, r, s, iters)
    lr_gpu = s * (host(B).astype(np.float64) @ host(A).astype(np.float64))
    lr_ref = s * (ref["B"].astype(np.float64) @ ref["A"].astype(np.float64))
    assert OL.rel_fro(lr_gpu, lr_ref) <= 1e-2
    # the quantised part: almost every code equal, and the same reconstruction quality
    got = _codes(host_bytes(q.codes), bits, N * K)
    exp = _codes(ref["q"]["packed"], bits, N * K)
    assert np.mean(got == exp) >= 0.99
    deq = host(cuda_lib.dequant(q)).astype(np.float64)
    err_gpu = np.linalg.norm(W - deq - lr_gpu) / np.linalg.norm(W)
    assert abs(err_gpu - ref["error"]) <= 0.05 * ref["error"] + 1e-4


def test_low_rank_dominated_matrix_beats_plain_quantisation(cuda_lib):
    N, K, r = 512, 1024, 32
    W = (random_matrix(7, 0, "A", (N, r), 1.0) @ random_matrix(7, 0, "B", (r, K), 1.0) * 0.02
         + random_matrix(7, 0, "W", (N, K), 0.005)).astype(np.float32)
    q0, _, _ = _run(cuda_lib, W, 2, 64, 256, r, 0.25, 0)
    q, A, B = _run(cuda_lib, W, 2, 64, 256, r, 0.25, 2)
    plain = np.linalg.norm(W - host(cuda_lib.dequant(q0))) / np.linalg.norm(W)
    recon = host(cuda_lib.dequant(q)).astype(np.float64) + 0.25 * (host(B).astype(np.float64) @ host(A).astype(np.float64))
    err = np.linalg.norm(W - recon) / np.linalg.norm(W)
    assert err < 0.5 * plain
