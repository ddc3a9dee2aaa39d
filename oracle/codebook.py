"""NF-k codebooks: quantile levels of the standard normal, normalised to [-1, 1] (oracle).

Source: QLoRA explainer, "Innovation 1: 4-bit NormalFloat (NF4)": 16 reconstruction
values placed so that every bin holds an equal share of a normal distribution,
used after dividing each block by its absolute maximum ("Background: what is
quantization?": normalise into the target range, then round to the nearest level).
LQ-LoRA (abstract) varies the bit width per matrix; the same construction with
2^k levels gives NF-2 / NF-3.

The listing on the QLoRA page places its levels at Phi^-1((i + 1/2) / 16); the page
calls that sketch simplified, and those levels contain no zero and span +-1.86,
which contradicts the normalisation to [-1, 1].  This oracle reads the levels as
the asymmetric quantile construction, which meets every property the page states:

  * 2^(k-1) positive levels Phi^-1(p) at p = the first 2^(k-1) of 2^(k-1)+1 evenly
    spaced points from delta down to 1/2;
  * 2^(k-1) - 1 negative levels -Phi^-1(p) at the first 2^(k-1) - 1 of 2^(k-1)
    evenly spaced points from delta down to 1/2;
  * an exact zero;
  * all divided by Phi^-1(delta), so the extremes are exactly -1 and +1.

delta (the outermost probability) is not on the pages; it is read as the mean of
the outermost bin centres of 2^k - 1 and 2^k equal-mass bins:
  delta_k = 1 - (1/(2 (2^k - 1)) + 1/(2 * 2^k)) / 2   (k=4: 0.9677083...).
Within each sign half, Phi(level * Phi^-1(delta)) is then evenly spaced: equal
probability mass per bin.
"""
from __future__ import annotations

import numpy as np
from scipy.stats import norm


def nf_delta(k: int) -> float:
    n = 2 ** k
    return 1.0 - 0.5 * (1.0 / (2.0 * (n - 1)) + 1.0 / (2.0 * n))


def nf_codebook(k: int) -> np.ndarray:
    """fp64 NF-k levels, ascending, length 2^k."""
    if k < 2 or k > 8:
        raise ValueError("k out of range")
    d = nf_delta(k)
    half = 2 ** (k - 1)
    pos = norm.ppf(np.linspace(d, 0.5, half + 1)[:-1])
    neg = -norm.ppf(np.linspace(d, 0.5, half)[:-1])
    levels = np.sort(np.concatenate([pos, neg, [0.0]]))
    return levels / norm.ppf(d)


def nf_codebook_f32(k: int) -> np.ndarray:
    """The levels as the quantiser and dequantiser use them: fp32(round-to-nearest of fp64)."""
    return nf_codebook(k).astype(np.float32)


def zero_index(k: int) -> int:
    return int(np.flatnonzero(nf_codebook_f32(k) == 0.0)[0])
