"""Pins of the LQ-LoRA initialisation oracle, each against something other than the oracle itself:
an SVD built by hand, an exactly low-rank matrix, plain quantisation at T = 0, the optimality
conditions of the second iteration's low-rank part, and the method's own
purpose (a strong low-rank component is reconstructed better than by quantisation alone)."""
import numpy as np

from oracle import lqlora as LQ
from oracle import quantize as Q


def _orthonormal(rng, n, k):
    q, _ = np.linalg.qr(rng.standard_normal((n, k)))
    return q[:, :k]


def test_first_iteration_low_rank_part_is_the_constructed_top_r_svd():
    rng = np.random.default_rng(0)
    N, K, r = 64, 96, 6
    U = _orthonormal(rng, N, N)
    V = _orthonormal(rng, K, N)
    sigma = np.linspace(3.0, 0.05, N) ** 2  # distinct, decreasing
    W = (U * sigma) @ V.T
    W32 = W.astype(np.float32)
    out = LQ.lqlora_init(W32, 4, 64, 256, r, 1.0, 1)
    # the oracle starts from Q = 0, so L_1 is the top-r part of fp32(W): the constructed triplets,
    # up to the fp32 rounding of W (relative 6e-8 of sigma_1, far below the gap between sigmas)
    expect = (U[:, :r] * sigma[:r]) @ V[:, :r].T
    assert np.linalg.norm(out["lowrank"] - expect) <= 1e-5 * np.linalg.norm(expect)


def test_exactly_low_rank_matrix_is_reconstructed_by_the_adapter():
    rng = np.random.default_rng(1)
    N, K, r = 48, 80, 8
    W = (rng.standard_normal((N, 5)) @ rng.standard_normal((5, K))).astype(np.float32)  # rank 5 <= r
    out = LQ.lqlora_init(W, 3, 64, 0, r, 0.5, 1)
    deq = Q.dequant_nfk(out["q"])
    # the residual after removing L_1 is rounding noise, so the quantised part is negligible ...
    assert np.abs(deq).max() <= 1e-5 * np.abs(W).max()
    # ... and s B A alone carries W, up to the bf16 rounding of the two factors
    assert out["error"] <= 1e-2


def test_zero_iterations_is_plain_quantisation_with_a_zero_adapter():
    rng = np.random.default_rng(2)
    W = (0.02 * rng.standard_normal((32, 128))).astype(np.float32)
    out = LQ.lqlora_init(W, 2, 128, 256, 4, 0.25, 0)
    ref = Q.quantize_nfk(W, 2, 128, 256)
    assert np.array_equal(out["q"]["packed"], ref["packed"])
    assert not out["A"].any() and not out["B"].any()


def test_strong_low_rank_component_beats_plain_quantisation():
    rng = np.random.default_rng(3)
    N, K, r = 128, 192, 8
    W = (rng.standard_normal((N, r)) @ rng.standard_normal((r, K)) * 0.05
         + 0.01 * rng.standard_normal((N, K))).astype(np.float32)
    plain = Q.dequant_nfk(Q.quantize_nfk(W, 2, 64, 256))
    err_plain = np.linalg.norm(W - plain) / np.linalg.norm(W)
    out = LQ.lqlora_init(W, 2, 64, 256, r, 0.25, 3)
    assert out["error"] < 0.5 * err_plain
    assert len(out["errors"]) == 3


def test_second_iteration_fits_the_residual_of_the_first():
    # L_2 must be the best rank-r approximation of W - dequant(Q_1), not of W: its residual E is
    # orthogonal to its own column and row spaces (the first-order condition of a truncated SVD), and
    # it fits that residual strictly better than L_1 does (Q_1 is far from zero at 2 bits)
    rng = np.random.default_rng(4)
    N, K, r = 64, 128, 4
    W = (rng.standard_normal((N, r)) @ rng.standard_normal((r, K)) * 0.03
         + 0.02 * rng.standard_normal((N, K))).astype(np.float32)
    one = LQ.lqlora_init(W, 2, 64, 0, r, 1.0, 1)
    two = LQ.lqlora_init(W, 2, 64, 0, r, 1.0, 2)
    R1 = W.astype(np.float64) - Q.dequant_nfk(one["q"]).astype(np.float64)
    L2 = two["lowrank"]
    E = R1 - L2
    col, _ = np.linalg.qr(L2 @ rng.standard_normal((K, r)))   # basis of L2's column space
    row, _ = np.linalg.qr(L2.T @ rng.standard_normal((N, r)))  # basis of its row space
    assert np.linalg.norm(col.T @ E) <= 1e-9 * np.linalg.norm(E)
    assert np.linalg.norm(E @ row) <= 1e-9 * np.linalg.norm(E)
    assert np.linalg.norm(E) < np.linalg.norm(R1 - one["lowrank"])
