"""Pins for the oracle's QWHA adapter initialisation and two-sided expansion (CPU only).

Expected values are worked by hand (allocations, top-k with ties), come from
brute force over every subset on tiny rows, or from closed forms: the outer
product of two popcount Hadamard columns, Parseval for an orthonormal
transform, the adjoint identity, and the one-dimensional least-squares
projection <a, b> / <a, a>.
"""
import itertools

import numpy as np
import pytest

from oracle import qwha as oq
from oracle import sparse as osp
from tests.test_oracle_hadamard import popcount_hadamard


@pytest.mark.parametrize("err,budget,k_min,n,want", [
    ([1.0, 3.0], 6, 1, 8, [2, 4]),                 # proportional, no remainder
    ([1.0, 1.0, 1.0], 7, 1, 8, [3, 2, 2]),          # 4/3 each: the spare unit goes to row 0
    ([2.0, 1.0, 1.0], 8, 1, 8, [4, 2, 2]),          # shares 2.5, 1.25, 1.25
    ([100.0, 1.0], 6, 1, 4, [4, 2]),                # row 0 capped at n, the rest re-split
    ([0.0, 0.0, 0.0, 0.0], 10, 2, 5, [3, 3, 2, 2]),  # no error anywhere: equal split
    ([5.0, 0.0, 1.0], 3, 1, 6, [1, 1, 1]),          # budget = rows * k_min
    ([1.0, 2.0], 8, 0, 4, [4, 4]),                  # budget = rows * n
])
def test_allocation_hand_cases(err, budget, k_min, n, want):
    got = oq.allocate(np.array(err), budget, k_min, n)
    assert got.tolist() == want


def test_allocation_invariants_random():
    rng = np.random.default_rng(4)
    for _ in range(50):
        rows = int(rng.integers(1, 40))
        n = int(rng.integers(4, 64))
        k_min = int(rng.integers(0, 3))
        e = np.abs(rng.standard_t(2.0, size=rows))
        budget = int(rng.integers(rows * k_min, rows * n + 1))
        k = oq.allocate(e, budget, k_min, n)
        assert k.sum() == budget and k.min() >= k_min and k.max() <= n
        # more error never gets fewer parameters, unless the row is already at the cap
        for a in range(rows):
            for b in range(rows):
                if e[a] > e[b] and k[b] < n:
                    assert k[a] >= k[b]


def test_allocation_rejects_impossible_budgets():
    with pytest.raises(ValueError):
        oq.allocate(np.ones(3), 2, 1, 8)
    with pytest.raises(ValueError):
        oq.allocate(np.ones(3), 25, 1, 8)


def test_topk_hand_cases_with_ties():
    f = np.array([[0.1, -0.5, 0.5, 0.2], [0.0, 0.0, 0.0, 0.0]])
    for k0, want0 in ((1, [1]), (2, [1, 2]), (3, [1, 2, 3]), (4, [0, 1, 2, 3])):
        off, cols = oq.select(f, [k0, 2])
        assert cols[off[0]:off[1]].tolist() == want0
        assert cols[off[1]:off[2]].tolist() == [0, 1]


def test_topk_keeps_the_most_energy_brute_force():
    rng = np.random.default_rng(6)
    n = 8
    f = rng.standard_normal((5, n))
    for k in range(n + 1):
        off, cols = oq.select(f, [k] * 5)
        for r in range(5):
            got = set(cols[off[r]:off[r + 1]].tolist())
            best = max(itertools.combinations(range(n), k), key=lambda s: sum(f[r, j] ** 2 for j in s))
            assert got == set(best)


def test_coefficients_and_channel_error():
    rng = np.random.default_rng(7)
    n = 16
    dw = rng.standard_normal((3, n))
    h = popcount_hadamard(n) / 4.0
    np.testing.assert_allclose(oq.coefficients(dw), dw @ h, rtol=0, atol=1e-14)
    # dW = F* H^-1 recovers dW: the coefficients expand back to the error itself
    np.testing.assert_allclose(oq.coefficients(dw) @ h, dw, rtol=0, atol=1e-13)
    x = rng.standard_normal((n, 5))
    want = np.array([np.sqrt(sum(sum(dw[r, i] * x[i, t] for i in range(n)) ** 2 for t in range(5))) for r in range(3)])
    np.testing.assert_allclose(oq.channel_error(dw, x), want, rtol=1e-13)
    np.testing.assert_allclose(oq.channel_error(dw), np.sqrt((dw ** 2).sum(1)), rtol=1e-14)


def test_direct_values_reconstruction_error_is_the_dropped_energy():
    rng = np.random.default_rng(8)
    n = 32
    dw = rng.standard_normal((4, n))
    f = oq.coefficients(dw)
    k = oq.allocate(oq.channel_error(dw), 40, 1, n)
    off, cols = oq.select(f, k)
    vals = oq.direct_values(f, off, cols)
    v, c = oq.to_fixed_width(off, cols, vals)
    approx = osp.expand(v[None], c[None], n, 1.0 / np.sqrt(n))[0]
    for r in range(4):
        kept = f[r, cols[off[r]:off[r + 1]]]
        np.testing.assert_allclose(np.sum((dw[r] - approx[r]) ** 2), np.sum(f[r] ** 2) - np.sum(kept ** 2),
                                   rtol=1e-10, atol=1e-12)


def test_refine_identity_activations_equals_direct_values():
    rng = np.random.default_rng(9)
    n = 16
    dw = rng.standard_normal((3, n))
    f = oq.coefficients(dw)
    off, cols = oq.select(f, [2, 5, 1])
    np.testing.assert_allclose(oq.refine_values(dw, np.eye(n), off, cols), oq.direct_values(f, off, cols),
                               rtol=0, atol=1e-12)


def test_refine_full_selection_is_exact():
    rng = np.random.default_rng(10)
    n = 8
    dw = rng.standard_normal((2, n))
    x = rng.standard_normal((n, 20))
    off, cols = oq.select(oq.coefficients(dw), [n, n])
    vals = oq.refine_values(dw, x, off, cols)
    v, c = oq.to_fixed_width(off, cols, vals)
    np.testing.assert_allclose(osp.expand(v[None], c[None], n, 1.0 / np.sqrt(n))[0], dw, rtol=0, atol=1e-12)


def test_refine_single_coefficient_is_the_projection():
    rng = np.random.default_rng(11)
    n, t = 16, 12
    dw = rng.standard_normal((1, n))
    x = rng.standard_normal((n, t))
    h = popcount_hadamard(n)
    for j in (0, 5, 15):
        off, cols = np.array([0, 1]), np.array([j], dtype=np.int32)
        a = [sum(h[j, i] / 4.0 * x[i, s] for i in range(n)) for s in range(t)]
        b = [sum(dw[0, i] * x[i, s] for i in range(n)) for s in range(t)]
        want = sum(p * q for p, q in zip(a, b)) / sum(p * p for p in a)
        np.testing.assert_allclose(oq.refine_values(dw, x, off, cols)[0], want, rtol=1e-12)


def test_refine_is_no_worse_than_direct_on_the_output_error():
    rng = np.random.default_rng(12)
    n, t = 32, 48
    dw = rng.standard_normal((6, n))
    x = rng.standard_normal((n, t)) * (1.0 + 10.0 * (np.arange(n) % 7 == 0))[:, None]
    f = oq.coefficients(dw)
    off, cols = oq.select(f, oq.allocate(oq.channel_error(dw, x), 30, 1, n))

    def out_err(vals):
        v, c = oq.to_fixed_width(off, cols, vals)
        approx = osp.expand(v[None], c[None], n, 1.0 / np.sqrt(n))[0]
        return np.sum(((dw - approx) @ x) ** 2)

    assert out_err(oq.refine_values(dw, x, off, cols)) <= out_err(oq.direct_values(f, off, cols)) * (1 + 1e-12)


def test_fixed_width_padding_expands_like_the_ragged_rows():
    n = 16
    off = np.array([0, 3, 4, 4, 6])
    cols = np.array([1, 5, 9, 2, 0, 15], dtype=np.int32)
    vals = np.array([0.5, -1.0, 2.0, 3.0, 0.25, -0.75])
    v, c = oq.to_fixed_width(off, cols, vals)
    assert v.shape == (4, 3)
    dense = np.zeros((4, n))
    for r in range(4):
        for k in range(off[r], off[r + 1]):
            dense[r, cols[k]] += vals[k]
    np.testing.assert_allclose(osp.expand(v[None], c[None], n, 0.25)[0], dense @ popcount_hadamard(n) * 0.25,
                               rtol=0, atol=1e-14)


def test_two_sided_single_coefficient_is_an_outer_product():
    m, n = 8, 16
    hm, hn = popcount_hadamard(m), popcount_hadamard(n)
    for r, k in ((0, 0), (3, 11), (7, 15)):
        vals = np.zeros((1, m, 1))
        cols = np.zeros((1, m, 1), dtype=np.int64)
        vals[0, r, 0] = 1.5
        cols[0, r, 0] = k
        got = oq.expand_two_sided(vals, cols, m, n)[0]
        want = 1.5 * np.outer(hm[:, r], hn[k, :]) / np.sqrt(m * n)
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)


def test_two_sided_parseval_and_adjoint():
    rng = np.random.default_rng(13)
    b, m, n, k = 2, 8, 32, 5
    vals = rng.standard_normal((b, m, k))
    cols = np.stack([np.stack([rng.choice(n, k, replace=False) for _ in range(m)]) for _ in range(b)])
    dense = oq.expand_two_sided(vals, cols, m, n)
    np.testing.assert_allclose(np.sum(dense ** 2), np.sum(vals ** 2), rtol=1e-12)
    g = rng.standard_normal((b, m, n))
    np.testing.assert_allclose(np.sum(dense * g), np.sum(vals * oq.gather_two_sided(g, cols)), rtol=1e-12)


def test_pins_reject_planted_mistakes():
    # selection by signed value instead of magnitude
    def select_signed(f, counts):
        f = np.asarray(f)
        off = np.concatenate([[0], np.cumsum(counts)])
        cols = np.concatenate([np.sort(np.argsort(-f[r], kind="stable")[: counts[r]]) for r in range(f.shape[0])])
        return off, cols.astype(np.int32)

    f = np.array([[0.1, -0.5, 0.5, 0.2]])
    assert select_signed(f, [2])[1].tolist() != [1, 2]

    # allocation rounded to nearest instead of floor + largest remainder
    def alloc_round(err, budget, k_min, n):
        e = np.asarray(err, float)
        return np.rint((budget - len(e) * k_min) * e / e.sum()).astype(int) + k_min

    assert alloc_round([1.0, 1.0, 1.0], 7, 1, 8).tolist() != [3, 2, 2]


def test_quantization_error_is_bounded_by_the_scales():
    # In the rotated basis the error is at most s/2 per element, and the rotation is orthogonal,
    # so ||dW_r||^2 <= sum over groups of group * (s_g / 2)^2.
    from oracle import hadamard as oh
    from oracle import quant as oqz
    import synth
    d = synth.qwha_init(rows=16, n=256, tokens=8, per_row=8)
    dw = oq.quantization_error(d["w"], d["signs"], 4, 32)
    sc = oqz.quantize(oh.rht_rows(d["w"], d["signs"]), 4, 32)["scales"].astype(np.float64)
    assert np.all(np.sum(dw ** 2, axis=1) <= np.sum(32 * (sc / 2) ** 2, axis=1) * (1 + 1e-6))
    assert np.all(np.sum(dw ** 2, axis=1) > 0)


def test_initialisation_pipeline_on_the_recipe():
    import synth
    d = synth.qwha_init(rows=32, n=128, tokens=64, per_row=8)
    dw = oq.quantization_error(d["w"], d["signs"], 4, 32)
    f = oq.coefficients(dw)
    k = oq.allocate(oq.channel_error(dw, d["x"]), d["budget"], d["k_min"], 128)
    assert k.sum() == d["budget"] and k.min() >= 1
    off, cols = oq.select(f, k)
    x = d["x"].astype(np.float64)

    def out_err(vals):
        v, c = oq.to_fixed_width(off, cols, vals)
        return np.sum(((dw - osp.expand(v[None], c[None], 128, 1.0 / np.sqrt(128))[0]) @ x) ** 2)

    base = np.sum((dw @ x) ** 2)
    direct = out_err(oq.direct_values(f, off, cols))
    refined = out_err(oq.refine_values(dw, x, off, cols))
    assert refined <= direct <= base
