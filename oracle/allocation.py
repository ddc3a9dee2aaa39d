"""LQ-LoRA's per-matrix choice of quantisation parameters under a memory budget (oracle; test
infrastructure).

LQ-LoRA (abstract): an integer linear programme picks each matrix's quantisation parameters (bit
width, block size) so that the whole model meets a memory budget.  Read as a multiple-choice knapsack: matrix i takes
exactly one option o (a bit width and block size) with reconstruction error err[i][o] (squared
Frobenius norm of W_i - dequant(Q_o(W_i))) and storage cost[i][o] (bits of its codes and constants);
minimise the summed error with the summed cost within the budget.

Solved exactly by dynamic programming over the budget in whole units of `unit` bits, each cost rounded
up to units (so the chosen plan never exceeds the budget): best[i][b] = min over o with c <= b of
best[i-1][b - c] + err[i][o], errors added in matrix order in float64.  The plan is read back from the
full budget, last matrix first, each taking the lowest option index among its minima; that resolves
ties between plans of equal total error.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

from .storage import nf_bytes


def nf_cost_bits(N: int, K: int, bits: int, block: int, dq_block: int) -> int:
    return 8 * sum(nf_bytes(N, K, bits, block, dq_block).values())


def squared_error(W: np.ndarray, Wdq: np.ndarray) -> float:
    d = np.asarray(W, np.float64) - np.asarray(Wdq, np.float64)
    return float(np.sum(d * d))


def allocate(err: Sequence[Sequence[float]], cost_bits: Sequence[Sequence[int]], budget_bits: int,
             unit: int) -> Tuple[List[int], float]:
    err = np.asarray(err, np.float64)
    m, n_opt = err.shape
    units = -(-np.asarray(cost_bits, np.int64) // unit)  # round up
    B = int(budget_bits // unit)
    inf = np.inf
    best = np.zeros(B + 1, np.float64)  # zero matrices: no error, any budget
    pick = np.zeros((m, B + 1), np.int16)
    for i in range(m):
        cand = np.full((n_opt, B + 1), inf)
        for o in range(n_opt):
            c = int(units[i, o])
            if c <= B:
                cand[o, c:] = best[: B + 1 - c] + err[i, o]
        pick[i] = np.argmin(cand, axis=0)
        best = cand[pick[i], np.arange(B + 1)]
    if not np.isfinite(best[B]):
        raise ValueError("budget below the cheapest plan")
    choice = [0] * m
    b = B
    for i in range(m - 1, -1, -1):
        o = int(pick[i, b])
        choice[i] = o
        b -= int(units[i, o])
    return choice, float(best[B])
