"""Randomized Walsh-Hadamard transform, dense and in float64 (test oracle only).

Definition followed (HARP explainer, technical summary §1 and §2.2; QWHA
explainer, technical summary §2.1): the Sylvester Hadamard matrix H_n has
entries +-1 and H_n H_n^T = n I; the randomized transform of a vector x of
length n is

    y = H_n diag(s) x / sqrt(n),        s in {+1, -1}^n,

which is orthogonal, so its inverse is x = diag(s) H_n y / sqrt(n).  Rows of a
matrix are transformed independently ("along rows", axis=1); "along columns"
(axis=0) applies the same map to every column.  The two-sided processor of
HARP §5 rotates both dimensions:

    W' = (H_m D_out / sqrt m) W (H_n D_in / sqrt n)^T.

Pinned by tests/test_oracle_hadamard.py: the popcount formula for the entries
(brute force, n <= 64), H H^T = n I, hand-worked n = 4 and n = 8 examples
(tests/golden/rht_hand_examples.txt), Parseval, inverse after forward, unit
vectors map to scaled Hadamard columns, and the two-sided form against explicit
dense matrix products.
"""
from __future__ import annotations

import numpy as np


def is_pow2(n: int) -> bool:
    return n >= 1 and (n & (n - 1)) == 0


def sylvester(n: int) -> np.ndarray:
    """H_n by the doubling recursion H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    if not is_pow2(n):
        raise ValueError(f"n={n} is not a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def _signs(s, n):
    if s is None:
        return np.ones(n, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64).reshape(-1)
    if s.shape[0] != n:
        raise ValueError("sign vector length must equal the transform length")
    return s


def rht_rows(x, signs=None) -> np.ndarray:
    """Forward transform of every row: y_r = H diag(s) x_r / sqrt(n), float64."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    h = sylvester(n)
    # H is symmetric, so the row-vector form of H D x is (x * s) @ H.
    return ((x * _signs(signs, n)) @ h) / np.sqrt(n)


def irht_rows(y, signs=None) -> np.ndarray:
    """Inverse transform of every row: x_r = diag(s) H y_r / sqrt(n), float64."""
    y = np.asarray(y, dtype=np.float64)
    n = y.shape[-1]
    h = sylvester(n)
    return ((y @ h) / np.sqrt(n)) * _signs(signs, n)


def rht_cols(x, signs=None) -> np.ndarray:
    """Forward transform of every column (transform length = number of rows)."""
    return rht_rows(np.asarray(x, dtype=np.float64).T, signs).T


def irht_cols(y, signs=None) -> np.ndarray:
    """Inverse transform of every column."""
    return irht_rows(np.asarray(y, dtype=np.float64).T, signs).T


def rht(x, signs=None, axis: int = 1, inverse: bool = False) -> np.ndarray:
    if axis == 1:
        return irht_rows(x, signs) if inverse else rht_rows(x, signs)
    if axis == 0:
        return irht_cols(x, signs) if inverse else rht_cols(x, signs)
    raise ValueError("axis must be 0 or 1")


def two_sided(w, row_signs, col_signs) -> np.ndarray:
    """W' = (H_m D_out / sqrt m) W (H_n D_in / sqrt n)^T with D_in = diag(row_signs)
    acting along each row (length n) and D_out = diag(col_signs) along each
    column (length m)."""
    return rht_cols(rht_rows(w, row_signs), col_signs)


def two_sided_inverse(wp, row_signs, col_signs) -> np.ndarray:
    """Inverse of :func:`two_sided`."""
    return irht_rows(irht_cols(wp, col_signs), row_signs)


def hadamard_rows(n: int, idx) -> np.ndarray:
    """Selected rows of H_n from the entry formula H[i, j] = (-1)^popcount(i & j)
    (the closed form of the Sylvester recursion; H is symmetric, so these are
    also its columns).  Used to evaluate sampled outputs of large transforms."""
    if not is_pow2(n):
        raise ValueError(f"n={n} is not a power of two")
    i = np.asarray(idx, dtype=np.int64)[:, None]
    v = i & np.arange(n, dtype=np.int64)[None, :]
    par = np.zeros(v.shape, dtype=np.int64)
    while np.any(v):
        par ^= v & 1
        v >>= 1
    return np.where(par == 1, -1.0, 1.0)


def rht_rows_at(x, signs, cols) -> np.ndarray:
    """Columns `cols` of the row-wise forward transform of x (float64)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    return ((x * _signs(signs, n)) @ hadamard_rows(n, cols).T) / np.sqrt(n)


def two_sided_rows_at(w, row_signs, col_signs, rows_idx) -> np.ndarray:
    """Rows `rows_idx` of two_sided(w, row_signs, col_signs): the column transform
    restricted to those output rows, then the full row transform."""
    w = np.asarray(w, dtype=np.float64)
    m = w.shape[0]
    z = ((hadamard_rows(m, rows_idx) * _signs(col_signs, m)) @ w) / np.sqrt(m)
    return rht_rows(z, row_signs)


def two_sided_inverse_rows_at(wp, row_signs, col_signs, rows_idx) -> np.ndarray:
    """Rows `rows_idx` of two_sided_inverse(wp, ...): the inverse column transform
    restricted to those rows, then the full inverse row transform."""
    wp = np.asarray(wp, dtype=np.float64)
    m = wp.shape[0]
    idx = np.asarray(rows_idx)
    z = (hadamard_rows(m, idx) @ wp) / np.sqrt(m) * _signs(col_signs, m)[idx][:, None]
    return irht_rows(z, row_signs)


def rht_rows_chunked(x, signs, chunk: int = 1024) -> np.ndarray:
    """rht_rows for long rows, building H_n a block of columns at a time."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    out = np.empty(x.shape, dtype=np.float64)
    for c0 in range(0, n, chunk):
        cols = np.arange(c0, min(n, c0 + chunk))
        out[..., cols] = rht_rows_at(x, signs, cols)
    return out


def irht_rows_chunked(y, signs, chunk: int = 1024) -> np.ndarray:
    """irht_rows for long rows, building H_n a block of columns at a time:
    output column j is (y . H[:, j]) / sqrt(n) * s_j (H is symmetric)."""
    y = np.asarray(y, dtype=np.float64)
    n = y.shape[-1]
    s = _signs(signs, n)
    out = np.empty(y.shape, dtype=np.float64)
    for c0 in range(0, n, chunk):
        cols = np.arange(c0, min(n, c0 + chunk))
        out[..., cols] = (y @ hadamard_rows(n, cols).T) / np.sqrt(n) * s[cols]
    return out
