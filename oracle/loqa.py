"""LoQA: gradients of the loss with respect to the quantiser's scale and zero point (oracle; test infrastructure).

Source: LoQA (OpenReview, abstract).  The abstract fine-tunes all the quantisation parameters of a
quantised model -- the scale and the zero point -- through a rewriting of the quantisation operator that
works with LoRA and computes the same thing as the original operator; it gives no formula.  This oracle
takes the plainest reading on the group-wise INT4 format the build already has (QA-LoRA abstract):

  * the dequantised weight is W[o, k] = s[o, g] (c[o, k] - z[o, g]),  g = k // L, with the integer
    codes c frozen and the per-(row, group) scale s and zero point z trainable;
  * the operator rewritten: with E spreading a per-group value over the group's L inputs and
    Psum(X)[m, g] = sum of X[m, k] over the group,
        X W^T = X (E(s) * C)^T - Psum(X) (s * z)^T,
    i.e. the zero point enters exactly like QA-LoRA's pooled adapter (a product with the group sums of
    the input), which is what makes it trainable alongside a LoRA adapter;
  * the layer's forward rounds W to bf16; the gradients pass that rounding straight through (it has
    no useful derivative), so with G = dY^T X (the gradient of the loss with respect to W):
        dL/ds[o, g] = sum_{k in g} G[o, k] (c[o, k] - z[o, g])
        dL/dz[o, g] = - s[o, g] sum_{k in g} G[o, k].

The LoRA scaling strategy of the abstract (a norm adjustment driven by quantisation statistics) is not
specified there and is not part of this module.

Everything is fp64; G is formed with one library matrix product.
"""
from __future__ import annotations

from typing import Dict

import numpy as np


def unrounded_weight(codes: np.ndarray, scale: np.ndarray, zero: np.ndarray, L: int) -> np.ndarray:
    """W[o, k] = s[o, k // L] (c[o, k] - z[o, k // L]) in fp64 (no bf16 rounding)."""
    c = np.asarray(codes, np.float64)
    N, K = c.shape
    s = np.repeat(np.asarray(scale, np.float64), L, axis=1)
    z = np.repeat(np.asarray(zero, np.float64), L, axis=1)
    assert s.shape == (N, K)
    return s * (c - z)


def group_sums(X: np.ndarray, L: int) -> np.ndarray:
    """Psum(X)[m, g] = sum over the L inputs of group g (fp64)."""
    X = np.asarray(X, np.float64)
    M, K = X.shape
    return X.reshape(M, K // L, L).sum(axis=-1)


def rewritten_product(X, codes, scale, zero, L: int) -> np.ndarray:
    """X W^T through the rewritten operator: X (E(s) * C)^T - Psum(X) (s * z)^T."""
    X = np.asarray(X, np.float64)
    s = np.asarray(scale, np.float64)
    sc = np.repeat(s, L, axis=1) * np.asarray(codes, np.float64)
    return X @ sc.T - group_sums(X, L) @ (s * np.asarray(zero, np.float64)).T


def scale_zero_grads(X, dY, codes, scale, zero, L: int) -> Dict[str, np.ndarray]:
    """dL/ds and dL/dz [N, K / L] for the loss whose gradient with respect to Y = X W^T is dY."""
    G = np.asarray(dY, np.float64).T @ np.asarray(X, np.float64)        # [N, K]
    N, K = G.shape
    c = np.asarray(codes, np.float64)
    z = np.asarray(zero, np.float64)
    Gg = G.reshape(N, K // L, L)
    cg = c.reshape(N, K // L, L)
    dscale = (Gg * (cg - z[..., None])).sum(axis=-1)
    dzero = -np.asarray(scale, np.float64) * Gg.sum(axis=-1)
    return {"dscale": dscale, "dzero": dzero, "G": G}
