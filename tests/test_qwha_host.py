"""AdaAlloc's budget split as the library computes it on the host
(qwha_allocate, through the C ABI), bit for bit against oracle.qwha.allocate
(CPU only: the split is host arithmetic on one number per row)."""
import numpy as np
import pytest

import hadamard_incoherence_transforms_b200 as hit
from hadamard_incoherence_transforms_b200 import _lib
from oracle import qwha as oqw


@pytest.fixture(scope="module", autouse=True)
def _built():
    import os

    if not os.path.exists(_lib.LIB_PATH):
        from hadamard_incoherence_transforms_b200 import build

        build.build()


def test_random_allocations_equal_the_oracle():
    rng = np.random.default_rng(20260)
    for trial in range(400):
        rows = int(rng.integers(1, 80))
        n = int(rng.choice([4, 8, 16, 64, 4096]))
        k_min = int(rng.integers(0, min(3, n) + 1))
        budget = int(rng.integers(rows * k_min, rows * n + 1))
        e = rng.random(rows) ** rng.choice([1, 4, 20])
        if trial % 7 == 0:
            e[:] = 0.0                       # equal split
        if trial % 5 == 0:
            e = np.round(e * 4) / 4          # exact ties in the fractional parts
        if trial % 11 == 0:
            e[0] = 1e6                       # a capped row, then a re-split
        got = hit.qwha_allocate(e, budget, k_min, n)
        want = oqw.allocate(e, budget, k_min, n)
        assert np.array_equal(got, want), (trial, rows, n, k_min, budget)
        assert int(got.sum()) == budget and got.min() >= k_min and got.max() <= n


def test_workload_sized_allocation():
    rng = np.random.default_rng(7)
    e = np.abs(rng.standard_normal(4096)) * 1e-2
    e[::97] *= 30.0
    got = hit.qwha_allocate(e, 64 * 4096, 1, 4096)
    assert np.array_equal(got, oqw.allocate(e, 64 * 4096, 1, 4096))


def test_bad_budgets_are_rejected():
    e = np.ones(4)
    for budget, k_min in ((3, 1), (4 * 16 + 1, 0)):
        with pytest.raises(_lib.HitError):
            hit.qwha_allocate(e, budget, k_min, 16)
    with pytest.raises(_lib.HitError):
        hit.qwha_allocate(np.array([1.0, -1.0]), 4, 1, 16)
    with pytest.raises(_lib.HitError):
        hit.qwha_allocate(np.array([1.0, np.nan]), 4, 1, 16)
