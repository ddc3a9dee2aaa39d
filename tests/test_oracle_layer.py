"""Pins for the fp64 forward/backward: scalar brute force on tiny shapes and
directional finite differences of the loss <Y, dY>."""
import numpy as np
import pytest

from oracle.layer import backward, forward, pool, swiglu_backward, swiglu_forward, unpool
from synth import random_matrix


def brute_forward(X, W, A, B, s, L=None):
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0]
    Ka = A.shape[1]
    Y = np.zeros((M, N))
    for m in range(M):
        p = [sum(float(X[m, g * L + j]) for j in range(L)) / L for g in range(Ka)] if L else [float(v) for v in X[m]]
        t = [sum(p[k] * float(A[j, k]) for k in range(Ka)) for j in range(r)]
        for n in range(N):
            base = sum(float(X[m, k]) * float(W[n, k]) for k in range(K))
            Y[m, n] = base + s * sum(t[j] * float(B[n, j]) for j in range(r))
    return Y


@pytest.mark.parametrize("L", [None, 4])
def test_forward_brute_force(L):
    M, K, N, r, s = 3, 8, 5, 2, 0.75
    X = random_matrix(1, 0, "X", (M, K), 1.0, True)
    W = random_matrix(1, 0, "W", (N, K), 0.5, True)
    A = random_matrix(1, 0, "A", (r, K // L if L else K), 0.5, True)
    B = random_matrix(1, 0, "B", (N, r), 0.5, True)
    np.testing.assert_allclose(forward(X, W, A, B, s, L)["Y"], brute_forward(X, W, A, B, s, L), rtol=1e-13, atol=1e-13)


def _loss(X, W, A, B, dY, s, L):
    return float(np.sum(forward(X, W, A, B, s, L)["Y"] * dY))


@pytest.mark.parametrize("L", [None, 32])
def test_backward_directional_finite_differences(L):
    M, K, N, r, s = 16, 256, 256, 8, 2.0       # the tiny workload's shape
    X = random_matrix(2, 0, "X", (M, K), 1.0, True).astype(np.float64)
    W = random_matrix(2, 0, "W", (N, K), 0.02, True).astype(np.float64)
    A = random_matrix(2, 0, "A", (r, K // L if L else K), 0.01, True).astype(np.float64)
    B = random_matrix(2, 0, "B", (N, r), 0.01, True).astype(np.float64)
    dY = random_matrix(2, 0, "dY", (M, N), 1.0, True).astype(np.float64)
    g = backward(dY, X, W, A, B, s, L)
    rng = np.random.default_rng(0)
    eps = 1e-3
    for name, grad in (("X", g["dX"]), ("A", g["dA"]), ("B", g["dB"])):
        for _ in range(3):
            args = {"X": X, "A": A, "B": B}
            V = rng.standard_normal(args[name].shape)
            plus = dict(args)
            minus = dict(args)
            plus[name] = args[name] + eps * V
            minus[name] = args[name] - eps * V
            fd = (_loss(plus["X"], W, plus["A"], plus["B"], dY, s, L)
                  - _loss(minus["X"], W, minus["A"], minus["B"], dY, s, L)) / (2 * eps)
            an = float(np.sum(grad * V))
            assert fd == pytest.approx(an, rel=1e-7, abs=1e-9), name


def test_pool_unpool_adjoint():
    X = random_matrix(3, 0, "X", (4, 64), 1.0)
    G = random_matrix(3, 1, "X", (4, 2), 1.0)
    assert float(np.sum(pool(X, 32) * G)) == pytest.approx(float(np.sum(X * unpool(G, 32))), rel=1e-12)
    np.testing.assert_allclose(pool(X, 32)[:, 0], X[:, :32].astype(np.float64).mean(axis=1), rtol=1e-15)


def test_swiglu_backward_finite_differences():
    G = random_matrix(4, 0, "X", (8, 16), 1.5)
    U = random_matrix(4, 1, "X", (8, 16), 1.0)
    dH = random_matrix(4, 2, "X", (8, 16), 1.0)
    dG, dU = swiglu_backward(dH, G, U)
    eps = 1e-5
    for grad, which in ((dG, 0), (dU, 1)):
        V = np.random.default_rng(which).standard_normal(G.shape)
        Gp, Up = (G + eps * V, U) if which == 0 else (G, U + eps * V)
        Gm, Um = (G - eps * V, U) if which == 0 else (G, U - eps * V)
        fd = (np.sum(swiglu_forward(Gp, Up) * dH) - np.sum(swiglu_forward(Gm, Um) * dH)) / (2 * eps)
        assert fd == pytest.approx(float(np.sum(grad * V)), rel=1e-7)
    # silu special values
    assert swiglu_forward(np.array([0.0]), np.array([1.0]))[0] == 0.0
    assert swiglu_forward(np.array([50.0]), np.array([1.0]))[0] == pytest.approx(50.0)
