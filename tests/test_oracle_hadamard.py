"""Pins for the oracle's randomized Hadamard transform (CPU only).

Each check rests on something other than the oracle's own code: the popcount
formula for Sylvester entries, orthogonality, hand-worked examples, Parseval,
and explicit dense matrix products built from the popcount formula.
"""
import numpy as np
import pytest

from oracle import hadamard as oh
from tests._golden import rht_cases


def popcount_hadamard(n):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    par = np.zeros((n, n), dtype=np.int64)
    v = i & j
    while np.any(v):
        par ^= v & 1
        v = v >> 1
    return np.where(par == 1, -1.0, 1.0)


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_sylvester_equals_popcount_formula(n):
    assert np.array_equal(oh.sylvester(n), popcount_hadamard(n))


@pytest.mark.parametrize("n", [2, 16, 256, 1024])
def test_hadamard_orthogonal_and_pm1(n):
    h = oh.sylvester(n)
    assert set(np.unique(h)) == {-1.0, 1.0}
    assert np.array_equal(h @ h.T, n * np.eye(n))


def test_rejects_non_power_of_two():
    for n in (0, 3, 12, 4095):
        with pytest.raises(ValueError):
            oh.sylvester(n)


@pytest.mark.parametrize("case", list(rht_cases()), ids=lambda c: f"n{c[0]}")
def test_hand_worked_examples(case):
    n, x, s, y = case
    got = oh.rht_rows(x[None, :], s)[0]
    np.testing.assert_allclose(got, y, rtol=0, atol=1e-15)
    back = oh.irht_rows(got[None, :], s)[0]
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [2, 8, 64, 512, 4096])
def test_parseval_and_inverse(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((5, n))
    s = rng.choice([-1, 1], size=n)
    y = oh.rht_rows(x, s)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oh.irht_rows(y, s), x, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [4, 32, 128])
def test_unit_vectors_give_scaled_hadamard_columns(n):
    rng = np.random.default_rng(7)
    s = rng.choice([-1, 1], size=n)
    h = popcount_hadamard(n)
    y = oh.rht_rows(np.eye(n), s)           # row k = transform of e_k
    expect = (s[:, None] * h.T) / np.sqrt(n)  # H D e_k = s_k * column k of H
    np.testing.assert_allclose(y, expect, rtol=0, atol=1e-15)


def test_linearity():
    rng = np.random.default_rng(3)
    n = 256
    s = rng.choice([-1, 1], size=n)
    a, b = rng.standard_normal((2, 3, n))
    np.testing.assert_allclose(oh.rht_rows(2.5 * a - b, s),
                               2.5 * oh.rht_rows(a, s) - oh.rht_rows(b, s), atol=1e-12)


@pytest.mark.parametrize("m,n", [(8, 16), (32, 4), (64, 64)])
def test_two_sided_matches_explicit_products(m, n):
    rng = np.random.default_rng(m * 1000 + n)
    w = rng.standard_normal((m, n))
    s_in = rng.choice([-1, 1], size=n)
    s_out = rng.choice([-1, 1], size=m)
    left = popcount_hadamard(m) @ np.diag(s_out) / np.sqrt(m)
    right = popcount_hadamard(n) @ np.diag(s_in) / np.sqrt(n)
    expect = left @ w @ right.T
    got = oh.two_sided(w, s_in, s_out)
    np.testing.assert_allclose(got, expect, atol=1e-12)
    np.testing.assert_allclose(oh.two_sided_inverse(got, s_in, s_out), w, atol=1e-12)
    # column transform alone is the left factor
    np.testing.assert_allclose(oh.rht_cols(w, s_out), left @ w, atol=1e-12)
    np.testing.assert_allclose(oh.irht_cols(left @ w, s_out), w, atol=1e-12)


@pytest.mark.parametrize("n", [1, 2, 64, 1024])
def test_hadamard_rows_equal_sylvester(n):
    idx = np.unique(np.random.default_rng(n).integers(0, n, size=min(n, 17)))
    assert np.array_equal(oh.hadamard_rows(n, idx), oh.sylvester(n)[idx])


def test_sampled_outputs_equal_full_transforms():
    rng = np.random.default_rng(21)
    m, n = 64, 256
    w = rng.standard_normal((m, n))
    s_in, s_out = rng.choice([-1, 1], n), rng.choice([-1, 1], m)
    cols = np.array([0, 5, 255])
    np.testing.assert_allclose(oh.rht_rows_at(w, s_in, cols), oh.rht_rows(w, s_in)[:, cols], atol=1e-12)
    rows = np.array([1, 30, 63])
    np.testing.assert_allclose(oh.two_sided_rows_at(w, s_in, s_out, rows), oh.two_sided(w, s_in, s_out)[rows],
                               atol=1e-12)


def test_sampled_inverse_and_chunked_forward():
    rng = np.random.default_rng(22)
    m, n = 32, 128
    wp = rng.standard_normal((m, n))
    s_in, s_out = rng.choice([-1, 1], n), rng.choice([-1, 1], m)
    rows = np.array([0, 7, 31])
    np.testing.assert_allclose(oh.two_sided_inverse_rows_at(wp, s_in, s_out, rows),
                               oh.two_sided_inverse(wp, s_in, s_out)[rows], atol=1e-12)
    np.testing.assert_allclose(oh.rht_rows_chunked(wp, s_in, chunk=48), oh.rht_rows(wp, s_in), atol=1e-12)
    np.testing.assert_allclose(oh.irht_rows_chunked(wp, s_in, chunk=48), oh.irht_rows(wp, s_in), atol=1e-12)


def test_chunked_inverse_undoes_chunked_forward():
    # signs after H on the inverse side: a sign error or a missing 1/sqrt(n)
    # breaks the round trip on rows long enough to need the chunked forms
    rng = np.random.default_rng(23)
    n = 4096
    x = rng.standard_normal((2, n))
    s = rng.choice([-1, 1], n)
    back = oh.irht_rows_chunked(oh.rht_rows_chunked(x, s, chunk=1000), s, chunk=777)
    np.testing.assert_allclose(back, x, atol=1e-10)
    # e_0 through the inverse is s * (first column of H) / sqrt(n)
    e0 = np.zeros((1, n))
    e0[0, 0] = 1.0
    np.testing.assert_allclose(oh.irht_rows_chunked(e0, s, chunk=999)[0], s / np.sqrt(n), atol=1e-15)
