"""The library's budgeted allocation (host code, no GPU) against the oracle's dynamic programme: the
same plan and the same total, tie rule included, and the documented argument errors."""
import numpy as np
import pytest

from oracle import allocation as AL


@pytest.fixture(scope="module")
def qlr():
    from quantized_base_lora_nf4_b200 import build, qlr as q
    build.build()
    q.lib()
    return q


@pytest.mark.parametrize("seed", range(8))
def test_same_plan_as_the_oracle(qlr, seed):
    rng = np.random.default_rng(100 + seed)
    m, n = int(rng.integers(1, 40)), int(rng.integers(1, 7))
    err = rng.uniform(0.0, 5.0, (m, n))
    err[rng.uniform(size=(m, n)) < 0.1] = 1.0  # some exact ties
    cost = rng.integers(1_000, 50_000, (m, n))
    unit = int(rng.choice([1, 7, 100, 1000]))
    lo, hi = int(cost.min(axis=1).sum()), int(cost.max(axis=1).sum())
    budget = int(rng.integers(lo + unit * m, hi + unit * m + 1))
    choice, total = qlr.lqlora_allocate(err, cost, budget, unit)
    ref_choice, ref_total = AL.allocate(err, cost, budget, unit)
    assert choice == ref_choice
    assert total == ref_total
    units = -(-cost // unit)
    assert sum(units[i, o] for i, o in enumerate(choice)) <= budget // unit


def test_errors(qlr):
    from quantized_base_lora_nf4_b200.qlr import QLRError
    err = np.ones((3, 2))
    cost = np.full((3, 2), 100, dtype=np.int64)
    with pytest.raises(QLRError) as e:  # below the cheapest plan
        qlr.lqlora_allocate(err, cost, 299, 1)
    assert e.value.code == -2
    with pytest.raises(QLRError) as e:  # too many budget units
        qlr.lqlora_allocate(err, cost, 1 << 40, 1)
    assert e.value.code == -2
    with pytest.raises(QLRError) as e:
        qlr.lqlora_allocate(err, cost, 1000, 0)
    assert e.value.code == -1
