"""Pins for the NF-k codebook: the invariants the QLoRA page states, checked with an
inverse normal computed here by bisection on math.erf (independent of scipy)."""
import math

import numpy as np
import pytest

from oracle.codebook import nf_codebook, nf_codebook_f32, nf_delta, zero_index


def phi(x: float) -> float:
    return 0.5 * (1.0 + math.erf(x / math.sqrt(2.0)))


def phi_inv(p: float) -> float:
    lo, hi = -40.0, 40.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if phi(mid) < p:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


@pytest.mark.parametrize("k", [2, 3, 4])
def test_level_count_order_range_zero(k):
    q = nf_codebook(k)
    assert q.size == 2 ** k                       # k=4: 16 reconstruction values
    assert np.all(np.diff(q) > 0)
    assert q[0] == -1.0 and q[-1] == 1.0          # normalised into [-1, 1] exactly
    assert np.count_nonzero(q == 0.0) == 1        # exact zero
    q32 = nf_codebook_f32(k)
    assert q32[0] == -1.0 and q32[-1] == 1.0 and q32[zero_index(k)] == 0.0


@pytest.mark.parametrize("k", [2, 3, 4])
def test_equal_probability_mass_per_bin(k):
    """Within each sign half, Phi(level * z_delta) is evenly spaced from 1/2 to delta."""
    q = nf_codebook(k)
    zd = phi_inv(nf_delta(k))
    pos = q[q >= 0]
    neg = -q[q <= 0][::-1]
    for half in (pos, neg):
        p = np.array([phi(v * zd) for v in half])
        steps = np.diff(p)
        assert p[0] == pytest.approx(0.5, abs=1e-15)
        assert p[-1] == pytest.approx(nf_delta(k), abs=1e-12)
        np.testing.assert_allclose(steps, steps[0], rtol=1e-9)
    assert pos.size == 2 ** (k - 1) + 1 and neg.size == 2 ** (k - 1)


@pytest.mark.parametrize("k", [2, 3, 4])
def test_levels_agree_with_bisection_quantiles(k):
    d = nf_delta(k)
    half = 2 ** (k - 1)
    ps = [d - i * (d - 0.5) / half for i in range(half)]
    ns = [d - i * (d - 0.5) / (half - 1) for i in range(half - 1)]
    zd = phi_inv(d)
    ref = sorted([phi_inv(p) / zd for p in ps] + [-phi_inv(p) / zd for p in ns] + [0.0])
    np.testing.assert_allclose(nf_codebook(k), ref, atol=1e-13)


def test_delta_k4():
    assert nf_delta(4) == pytest.approx(1 - 0.5 * (1 / 30 + 1 / 32), abs=0)
    assert nf_delta(4) == pytest.approx(0.9677083333, abs=1e-10)


def test_sketch_levels_contradict_normalisation():
    """The page's simplified listing uses Phi^-1((i+1/2)/16): no zero, extremes beyond 1.
    This is why the oracle takes the quantile construction that meets the stated invariants."""
    sketch = np.array([phi_inv((i + 0.5) / 16) for i in range(16)])
    assert np.count_nonzero(np.abs(sketch) < 1e-12) == 0
    assert sketch.max() > 1.8
