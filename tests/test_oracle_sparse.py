"""Pins for the oracle's WHT expansion of sparse coefficients (CPU only)."""
import numpy as np
import pytest
import torch

from oracle import sparse as osp
from tests.test_oracle_hadamard import popcount_hadamard


def test_single_nonzero_closed_form():
    n, scale = 64, 1.0 / 8.0
    h = popcount_hadamard(n)
    for k in (0, 1, 37, 63):
        v = np.array([[[2.5]]])
        c = np.array([[[k]]])
        got = osp.expand(v, c, n, scale)[0, 0]
        np.testing.assert_allclose(got, 2.5 * h[k] * scale, atol=1e-15)


def test_duplicates_add():
    n = 16
    v = np.array([[[1.0, 2.0, -0.5]]])
    c = np.array([[[3, 3, 9]]])
    f = osp.scatter_dense(v, c, n)[0, 0]
    assert f[3] == 3.0 and f[9] == -0.5 and np.count_nonzero(f) == 2


def test_adjoint_identity():
    rng = np.random.default_rng(1)
    b, r, n, k = 2, 5, 128, 7
    v = rng.standard_normal((b, r, k))
    c = np.stack([np.stack([rng.choice(n, k, replace=False) for _ in range(r)]) for _ in range(b)])
    g = rng.standard_normal((b, r, n))
    lhs = np.sum(osp.expand(v, c, n, 0.125) * g)
    rhs = np.sum(v * osp.gather_grad(g, c, 0.125))
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12)


def test_gradient_against_torch_autograd():
    rng = np.random.default_rng(2)
    b, r, n, k = 1, 3, 32, 4
    v = rng.standard_normal((b, r, k))
    c = rng.integers(0, n, size=(b, r, k))
    c[0, 0, 1] = c[0, 0, 0]                     # include a duplicate
    g = rng.standard_normal((b, r, n))
    h = torch.tensor(popcount_hadamard(n))
    vt = torch.tensor(v, requires_grad=True)
    f = torch.zeros((b, r, n), dtype=torch.float64).scatter_add(2, torch.tensor(c), vt)
    loss = ((f @ h) * 0.25 * torch.tensor(g)).sum()
    loss.backward()
    np.testing.assert_allclose(osp.gather_grad(g, c, 0.25), vt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(osp.expand(v, c, n, 0.25), ((f @ h) * 0.25).detach().numpy(), atol=1e-12)


def test_rejects_out_of_range_columns():
    with pytest.raises(ValueError):
        osp.scatter_dense(np.ones((1, 1, 1)), np.array([[[16]]]), 16)
