"""Pins of the budgeted bit-width / block-size allocation oracle: exhaustive search on small
instances, the two closed-form ends of the budget, and the storage cost formula."""
import itertools

import numpy as np
import pytest

from oracle import allocation as AL


def _brute(err, units, B):
    best, arg = np.inf, None
    m, n = err.shape
    for combo in itertools.product(range(n), repeat=m):
        c = sum(units[i][o] for i, o in enumerate(combo))
        if c <= B:
            e = sum(err[i][o] for i, o in enumerate(combo))
            if e < best:
                best, arg = e, combo
    return list(arg), best


@pytest.mark.parametrize("seed", range(6))
def test_dynamic_programme_matches_exhaustive_search(seed):
    rng = np.random.default_rng(seed)
    m, n = 5, 6
    err = rng.uniform(0.1, 10.0, (m, n))
    units = rng.integers(1, 20, (m, n))
    lo, hi = units.min(axis=1).sum(), units.max(axis=1).sum()
    B = int(rng.integers(lo, hi + 1))
    choice, total = AL.allocate(err, units, B, 1)
    ref_choice, ref_total = _brute(err, units, B)
    assert abs(total - ref_total) <= 1e-12 * ref_total
    assert choice == ref_choice
    assert sum(units[i][o] for i, o in enumerate(choice)) <= B


def test_budget_ends_have_closed_forms():
    rng = np.random.default_rng(9)
    err = rng.uniform(0.1, 10.0, (7, 6))
    cost = rng.integers(100, 2000, (7, 6))
    # unlimited budget: every matrix takes its smallest error
    choice, _ = AL.allocate(err, cost, int(cost.sum()), 1)
    assert choice == list(np.argmin(err, axis=1))
    # the cheapest plan's budget: every matrix takes its cheapest option (unique here)
    choice, _ = AL.allocate(err, cost, int(cost.min(axis=1).sum()), 1)
    assert choice == list(np.argmin(cost, axis=1))
    with pytest.raises(ValueError):
        AL.allocate(err, cost, int(cost.min(axis=1).sum()) - 1, 1)


def test_cost_rounding_never_exceeds_the_budget():
    err = np.array([[1.0, 2.0], [1.0, 2.0]])
    cost = np.array([[150, 100], [150, 100]])
    # 290 bits in units of 100 is 2 units; the 150-bit option rounds up to 2, so no plan with it fits
    choice, _ = AL.allocate(err, cost, 290, 100)
    assert choice == [1, 1]
    # in exact bits one matrix can take the better option (150 + 100 <= 290); the two plans tie, and
    # the read-back from the last matrix gives it the lowest option index
    choice, total = AL.allocate(err, cost, 290, 1)
    assert choice == [1, 0] and total == 3.0


def test_storage_cost_matches_the_closed_form():
    N = K = 4096
    for bits, block in ((4, 64), (3, 128), (2, 64)):
        expect = N * K * bits + N * K // block * 8 + N * K // (block * 256) * 32
        assert AL.nf_cost_bits(N, K, bits, block, 256) == expect
    assert AL.nf_cost_bits(N, K, 4, 64, 0) == N * K * 4 + N * K // 64 * 32
