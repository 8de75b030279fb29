"""Walsh-Hadamard expansion of sparse adapter coefficients, in float64 (test
oracle only).

QWHA explainer, technical summary §2.1: the adapter is dW = F H^-1 with H the
Walsh-Hadamard transform and F a sparse trainable coefficient matrix built
from a value vector c and an index list E; §4 credits scatter operations for
its low memory.  Reading: H^-1 is the orthonormal inverse, so along each row
dW_r = F_r H_n * scale with scale = 1/sqrt(n) (1/64 at n = 4096), F is stored
as [batch, rows, nnz] values plus int32 column indices, and duplicate column
indices in a row add up (scatter-add).  The gradient with respect to the
stored values is the adjoint: grad_c[b, r, k] = (G_r H_n * scale)[E[b, r, k]].

Pinned by tests/test_oracle_sparse.py: a single nonzero gives c * H[k, :] *
scale (popcount formula), duplicates sum, the adjoint identity
<expand(v), G> = <v, gather(G)>, and the gradient against exact finite
differences on a tiny case.
"""
from __future__ import annotations

import numpy as np

from .hadamard import sylvester


def scatter_dense(values, cols, n: int) -> np.ndarray:
    """F as a dense [batch, rows, n] float64 array (duplicates add)."""
    values = np.asarray(values, dtype=np.float64)
    cols = np.asarray(cols, dtype=np.int64)
    if values.shape != cols.shape or values.ndim != 3:
        raise ValueError("values and cols must both be [batch, rows, nnz]")
    if cols.size and (cols.min() < 0 or cols.max() >= n):
        raise ValueError("column index out of range")
    bsz, rows, nnz = values.shape
    f = np.zeros((bsz, rows, n), dtype=np.float64)
    b, r, _ = np.indices(values.shape)
    np.add.at(f, (b, r, cols), values)
    return f


def expand(values, cols, n: int, scale: float) -> np.ndarray:
    """dW[b, r, :] = scatter(values, cols)[b, r, :] @ H_n * scale."""
    return (scatter_dense(values, cols, n) @ sylvester(n)) * scale


def gather_grad(grad, cols, scale: float) -> np.ndarray:
    """grad_c[b, r, k] = (grad[b, r, :] @ H_n * scale)[cols[b, r, k]]."""
    grad = np.asarray(grad, dtype=np.float64)
    n = grad.shape[-1]
    full = (grad @ sylvester(n)) * scale
    return np.take_along_axis(full, np.asarray(cols, dtype=np.int64), axis=-1)
