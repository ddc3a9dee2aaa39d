"""Pins of the LoQA oracle (LoQA abstract: scale and zero point fine-tuned through a rewritten quantisation
operator that works with LoRA and computes the same thing as the original one).

* the rewritten operator reproduces X W^T for the dequantised INT4 weight (the "same thing" of the
  abstract), in fp64, on the oracle's own quantiser output;
* the gradients equal central finite differences of <X W(s, z)^T, dY>: the loss is linear in s for fixed
  z and in z for fixed s, so the differences are exact up to fp64 rounding;
* brute force with scalar loops on a tiny case;
* a zero point shifted by delta moves Y exactly like QA-LoRA's pooled adapter with A, B chosen to carry
  -s delta L, which ties the zero-point gradient to the merge identity the QA-LoRA pins already check.
"""
import numpy as np
import pytest

from oracle import layer as OL
from oracle import loqa as LQ
from oracle import quantize as Q
from synth import random_matrix


def _case(N=12, K=64, L=32, M=5, seed=0):
    W = random_matrix(40 + seed, 0, "W", (N, K), 0.02)
    q = Q.quantize_int4_group(W, L)
    codes = q["codes"].reshape(N, K)
    X = random_matrix(40 + seed, 1, "X", (M, K), 1.0, bf16=True)
    dY = random_matrix(40 + seed, 2, "dY", (M, N), 1.0, bf16=True)
    return q, codes, X, dY


def test_rewritten_operator_equals_the_original():
    q, codes, X, _ = _case()
    L = q["group"]
    W = LQ.unrounded_weight(codes, q["scale"], q["zero"], L)
    ref = np.asarray(X, np.float64) @ W.T
    got = LQ.rewritten_product(X, codes, q["scale"], q["zero"], L)
    assert np.max(np.abs(got - ref)) <= 1e-12 * np.max(np.abs(ref))
    # and the unrounded weight is the INT4 dequant before its bf16 rounding
    Wbf = Q.dequant_int4_group(q).astype(np.float64)
    assert np.max(np.abs(Wbf - W)) <= 2.0 ** -8 * np.max(np.abs(W))


def _loss(X, dY, codes, s, z, L):
    return float(np.sum((np.asarray(X, np.float64) @ LQ.unrounded_weight(codes, s, z, L).T) * dY))


@pytest.mark.parametrize("seed", [0, 1])
def test_gradients_match_finite_differences(seed):
    q, codes, X, dY = _case(seed=seed)
    L = q["group"]
    s = q["scale"].astype(np.float64)
    z = q["zero"].astype(np.float64)
    g = LQ.scale_zero_grads(X, dY, codes, s, z, L)
    h = 1e-3
    for (o, gg) in [(0, 0), (3, 1), (11, 0), (7, 1)]:
        e = np.zeros_like(s)
        e[o, gg] = h
        fd_s = (_loss(X, dY, codes, s + e, z, L) - _loss(X, dY, codes, s - e, z, L)) / (2 * h)
        fd_z = (_loss(X, dY, codes, s, z + e, L) - _loss(X, dY, codes, s, z - e, L)) / (2 * h)
        assert abs(fd_s - g["dscale"][o, gg]) <= 1e-8 * (1 + abs(fd_s))
        assert abs(fd_z - g["dzero"][o, gg]) <= 1e-8 * (1 + abs(fd_z))


def test_brute_force_tiny():
    q, codes, X, dY = _case(N=3, K=64, L=32, M=2, seed=3)
    L = q["group"]
    s, z = q["scale"].astype(np.float64), q["zero"].astype(np.float64)
    g = LQ.scale_zero_grads(X, dY, codes, s, z, L)
    for o in range(3):
        for gg in range(2):
            ds = dz = 0.0
            for k in range(gg * L, gg * L + L):
                gk = sum(float(dY[m, o]) * float(X[m, k]) for m in range(2))
                ds += gk * (float(codes[o, k]) - z[o, gg])
                dz += -s[o, gg] * gk
            assert abs(ds - g["dscale"][o, gg]) <= 1e-12 * (1 + abs(ds))
            assert abs(dz - g["dzero"][o, gg]) <= 1e-12 * (1 + abs(dz))


def test_zero_point_shift_is_a_pooled_adapter():
    """Shifting z by delta adds -s delta (sum over the group) to every output: the pooled adapter of
    QA-LoRA with T = mean over the group, A = identity on groups and B = -s delta L."""
    q, codes, X, _ = _case(N=8, K=128, L=32, M=4, seed=5)
    L = q["group"]
    s, z = q["scale"].astype(np.float64), q["zero"].astype(np.float64)
    delta = random_matrix(45, 0, "W", s.shape, 0.5)
    base = np.asarray(X, np.float64) @ LQ.unrounded_weight(codes, s, z, L).T
    shifted = np.asarray(X, np.float64) @ LQ.unrounded_weight(codes, s, z + delta, L).T
    G = s.shape[1]
    # pooled adapter y += s_lora (pool(X) A^T) B^T with A = I [G, G], B = -s delta L, s_lora = 1
    via_adapter = OL.forward(X, np.zeros_like(codes, dtype=np.float64), np.eye(G), -s * delta * L, 1.0, L)["Y"]
    assert np.max(np.abs((shifted - base) - via_adapter)) <= 1e-12 * (1 + np.max(np.abs(via_adapter)))
