"""Forward and backward of the quantised-base + LoRA linear, in fp64 (oracle; test infrastructure).

Sources:
  * QLoRA explainer, "Background: how LoRA works": W0 stays frozen, the update is
    Delta W = B A with B (d x r) and A (r x d), and the layer computes W0 x + B A x.
  * "The QLoRA recipe: quantize, then adapt", stage 3, and "The complete QLoRA
    forward pass": the frozen block is dequantised to bf16, multiplied by the input,
    and the LoRA correction is added; gradients reach only A and B.  The page's
    formula was lost in extraction; the code sketch computes x W^T + (x A^T) B^T.
    With the LoRA scale s:   Y = X W_dq^T + s (X A^T) B^T.
  * QA-LoRA abstract: the adapter sees fewer degrees of freedom; read as the adapter
    input being the mean of each group of L consecutive input channels.

Operands are the bf16 values (X, A, B, W_dq) held in fp64; every product and sum
is fp64.  Row-major: X [M, K], W [N, K], A [r, K_a], B [N, r], Y [M, N].

Backward of Y = X W^T + s T B^T with T = P(X) A^T (P = identity or group mean):
  dT = s dY B,   dB = s dY^T T,   dA = dT^T P(X),
  dX = dY W + P^T(dT A)   where P^T spreads each pooled column back over its
  L inputs with weight 1/L.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np


def f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def pool(X: np.ndarray, L: int) -> np.ndarray:
    """Group mean over L consecutive input channels: [M, K] -> [M, K / L]."""
    X = f64(X)
    M, K = X.shape
    return X.reshape(M, K // L, L).mean(axis=-1)


def unpool(G: np.ndarray, L: int) -> np.ndarray:
    """Adjoint of pool: every pooled column spread over its L inputs with weight 1/L."""
    return np.repeat(f64(G), L, axis=1) / L


def forward(X, Wdq, A, B, s: float, L: Optional[int] = None, dtype=np.float64) -> Dict[str, np.ndarray]:
    """dtype: the precision of the products (fp64 for parity; the timed CPU baseline passes fp32)."""
    X, Wdq, A, B = (np.asarray(a, dtype) for a in (X, Wdq, A, B))
    P = (pool(X, L).astype(dtype) if L else X)
    T = P @ A.T
    Y = X @ Wdq.T + s * (T @ B.T)
    return {"Y": Y, "T": T}


def backward(dY, X, Wdq, A, B, s: float, L: Optional[int] = None, dtype=np.float64) -> Dict[str, np.ndarray]:
    dY, X, Wdq, A, B = (np.asarray(a, dtype) for a in (dY, X, Wdq, A, B))
    P = (pool(X, L).astype(dtype) if L else X)
    T = P @ A.T
    dT = s * (dY @ B)
    dB = s * (dY.T @ T)
    dA = dT.T @ P
    dTA = dT @ A
    dX = dY @ Wdq + (unpool(dTA, L).astype(dtype) if L else dTA)
    return {"dX": dX, "dA": dA, "dB": dB, "dT": dT, "T": T}


def silu(g: np.ndarray) -> np.ndarray:
    g = f64(g)
    return g / (1.0 + np.exp(-g))


def swiglu_forward(G, U) -> np.ndarray:
    """H = silu(G) * U (the MLP block's gate between the up and down projections)."""
    return silu(G) * f64(U)


def swiglu_backward(dH, G, U):
    """dG = dH U sigma(G) (1 + G (1 - sigma(G))),  dU = dH silu(G)."""
    dH, G, U = f64(dH), f64(G), f64(U)
    sig = 1.0 / (1.0 + np.exp(-G))
    dG = dH * U * sig * (1.0 + G * (1.0 - sig))
    dU = dH * G * sig
    return dG, dU


def rel_fro(a, b) -> float:
    """||a - b||_F / ||b||_F (b is the oracle)."""
    a, b = f64(a), f64(b)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))
