"""LQ-LoRA initialisation (oracle; test infrastructure).

LQ-LoRA (abstract): an iterative method splits each pretrained matrix into a low-rank part kept in
high precision plus a quantised part that is cheap to store; during finetuning the quantised part
stays fixed and only the low-rank component (the adapter) is trained.  The abstract gives
no further steps; the reading used here is the plain alternation between the two components:

    Q_0 = 0
    for t = 1 .. T:
        L_t = best rank-r approximation of (W - dequant(Q_{t-1}))     (truncated SVD, Eckart-Young)
        Q_t = NF-k quantisation of fp32(W - L_t)                        (blockwise + double quant)

and the adapter of the layer h = dequant(Q) x + s B (A x) carries L_T:
    L_T = U_r diag(sigma_r) V_r^T,  A = bf16(diag(sqrt sigma_r) V_r^T),  B = bf16(U_r diag(sqrt sigma_r) / s),
so that s B A reproduces L_T up to the bf16 rounding of the factors.  T = 0 is plain quantisation
(A = B = 0).  Residuals and the SVD are fp64; the quantiser takes the fp32-rounded residual, as
the library's does.  The SVD is numpy's (a library primitive); singular vectors are unique only up
to sign, so only products such as L_T = s B A are comparable across implementations.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from . import quantize as Q
from .numerics import bf16_rn


def lqlora_init(W: np.ndarray, bits: int, block: int, dq_block: int, r: int, s: float, iters: int) -> Dict[str, object]:
    W64 = np.asarray(W, dtype=np.float32).astype(np.float64)
    N, K = W64.shape
    if not 1 <= r <= min(N, K):
        raise ValueError("rank out of range")
    deq = np.zeros_like(W64)
    lowrank = np.zeros_like(W64)
    q = None
    errors = []
    Ur = Sr = Vtr = None
    for _ in range(iters):
        U, S, Vt = np.linalg.svd(W64 - deq, full_matrices=False)
        Ur, Sr, Vtr = U[:, :r], S[:r], Vt[:r]
        lowrank = (Ur * Sr) @ Vtr
        q = Q.quantize_nfk((W64 - lowrank).astype(np.float32), bits, block, dq_block)
        deq = Q.dequant_nfk(q).astype(np.float64)
        errors.append(float(np.linalg.norm(W64 - deq - lowrank) / np.linalg.norm(W64)))
    if iters == 0:
        q = Q.quantize_nfk(W64.astype(np.float32), bits, block, dq_block)
        deq = Q.dequant_nfk(q).astype(np.float64)
        A = np.zeros((r, K), np.float32)
        B = np.zeros((N, r), np.float32)
    else:
        root = np.sqrt(Sr)
        A = bf16_rn((root[:, None] * Vtr).astype(np.float32))
        B = bf16_rn((Ur * root / s).astype(np.float32))
    W_hat = deq + s * (B.astype(np.float64) @ A.astype(np.float64))
    return {"q": q, "A": A, "B": B, "lowrank": lowrank, "W_hat": W_hat, "errors": errors,
            "error": float(np.linalg.norm(W64 - W_hat) / np.linalg.norm(W64))}
