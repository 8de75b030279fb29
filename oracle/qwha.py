"""QWHA's adapter initialisation around the sparse WHT expansion, in float64
(test oracle only).

QWHA explainer, technical summary §2.1: the single-transform adapter is
dW = F H^-1; the two-transform form other Fourier adapters use is
dW = H'^-1 F H^-1.  §2.2: AdaAlloc spreads a parameter budget p over the output
channels in proportion to the size of each channel's activation error, keeps a
minimum count per channel so the adapter stays full rank, and inside a channel
keeps the coefficients of largest magnitude; Refinement then fits the values c
on the chosen positions by least squares on the layer output error
||dW_Q X - F H^-1 X||_F^2.

Readings taken where the pages stop:

* H^-1 (and H'^-1) is the orthonormal inverse H_n / sqrt(n), which is its own
  inverse, so the dense coefficients of an error dW are F* = dW H_n / sqrt(n),
  row by row.
* A channel is a row of dW (an output channel).  Its activation error is
  e_r = ||(dW X)_r||_2 for activations X [n, T]; with no X it is ||dW_r||_2.
* Allocation: every row gets k_min; the remaining R = p - rows * k_min is split
  in proportion to e_r with no row above n: rows whose share would pass n are
  set to n and the rest re-split, until none passes; the shares are rounded
  down and the units left over go one each to the largest fractional parts
  (ties to the lower row).  If every uncapped e_r is zero the split is equal.
  The share of row r is (R' * e_r) / S in float64, with R' the units left for
  the uncapped rows and S the sum of their errors taken left to right in
  float64 (a fixed order, so any implementation can reproduce the split).
* Selection inside a row: the k_r largest |F*_{r,j}|, ties to the lower j; the
  chosen columns are returned in ascending order.
* Direct values: c = F*[r, E_r].  Refined values: per row, the least-squares
  solution of min_c ||X^T dW_r^T - X^T (H_n[E_r, :] / sqrt n)^T c||.
* The error matrix is that of the rotated quantizer: dW = W - W_hat, W_hat the
  inverse RHT of the dequantized codes of RHT(W).
* Ragged rows are stored CSR-style (offsets [rows + 1], columns, values); the
  fixed-width [rows, k_max] form pads a row with zero values on its first
  chosen column, which the scatter-add expansion leaves unchanged.
* The two-sided expansion is dense = (H_m / sqrt m) scatter(c, E) (H_n / sqrt n)
  for an [m, n] coefficient matrix, per batch.

Pinned by tests/test_oracle_qwha.py: a single coefficient expands to the outer
product of two popcount Hadamard columns; Parseval for the two-sided form and
its adjoint gather; hand-worked allocations (proportional, remainders, the
cap); hand-worked top-k with ties; brute force over every subset on tiny rows
(the chosen set keeps the most energy); refinement with X = I equal to the
direct values, a full selection reproducing dW exactly, and a one-coefficient
case against the closed-form projection.
"""
from __future__ import annotations

import numpy as np

from .hadamard import irht_rows, rht_rows, sylvester
from .quant import dequantize, quantize
from .sparse import scatter_dense


def quantization_error(w, signs, bits: int, group: int) -> np.ndarray:
    """dW = W - W_hat with W_hat = inverse RHT of the dequantized codes of RHT(W)."""
    w = np.asarray(w, dtype=np.float64)
    r = quantize(rht_rows(w, signs), bits, group)
    return w - irht_rows(dequantize(r["u"], r["scales"], bits, group), signs)


def coefficients(dw) -> np.ndarray:
    """F* = dW H_n / sqrt(n) for every row of dW [rows, n]."""
    dw = np.asarray(dw, dtype=np.float64)
    n = dw.shape[-1]
    return dw @ sylvester(n) / np.sqrt(n)


def channel_error(dw, x=None) -> np.ndarray:
    """e_r = ||(dW X)_r||_2, or ||dW_r||_2 without activations."""
    dw = np.asarray(dw, dtype=np.float64)
    out = dw if x is None else dw @ np.asarray(x, dtype=np.float64)
    return np.sqrt(np.sum(out * out, axis=-1))


def _sum_left_to_right(v) -> float:
    """sum(v) in float64, one element after the other from the first."""
    acc = 0.0
    for x in np.asarray(v, dtype=np.float64).tolist():
        acc += x
    return acc


def allocate(err, budget: int, k_min: int, n: int) -> np.ndarray:
    """Per-row counts k_r (int64) summing to budget, each in [k_min, n]."""
    e = np.asarray(err, dtype=np.float64)
    rows = e.shape[0]
    if k_min < 0 or k_min > n or budget < rows * k_min or budget > rows * n:
        raise ValueError("budget must lie in [rows * k_min, rows * n]")
    room = n - k_min
    left = budget - rows * k_min
    capped = np.zeros(rows, dtype=bool)
    while True:
        free = ~capped
        rest = left - room * int(capped.sum())
        w = e[free]
        if _sum_left_to_right(w) <= 0:
            w = np.ones_like(w)
        share = np.zeros(rows)
        share[free] = (float(rest) * w) / _sum_left_to_right(w)
        over = free & (share > room)
        if not over.any():
            break
        capped |= over
    share[capped] = room
    k = np.floor(share).astype(np.int64)
    k[capped] = room
    spare = left - int(k.sum())
    frac = share - np.floor(share)
    order = [r for r in sorted(range(rows), key=lambda r: (-frac[r], r)) if not capped[r] and k[r] < room]
    for r in order[:spare]:
        k[r] += 1
    return k + k_min


def select(f, counts):
    """CSR (offsets, cols) of the counts[r] largest |F_r| per row, ties to the lower column."""
    f = np.asarray(f, dtype=np.float64)
    rows, n = f.shape
    counts = np.asarray(counts, dtype=np.int64)
    offsets = np.zeros(rows + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    cols = np.empty(int(offsets[-1]), dtype=np.int32)
    for r in range(rows):
        order = np.lexsort((np.arange(n), -np.abs(f[r])))
        cols[offsets[r]:offsets[r + 1]] = np.sort(order[: counts[r]])
    return offsets, cols


def direct_values(f, offsets, cols) -> np.ndarray:
    """c = F*[r, E_r] on the CSR layout."""
    f = np.asarray(f, dtype=np.float64)
    rows = f.shape[0]
    row_of = np.repeat(np.arange(rows), np.diff(offsets))
    return f[row_of, cols]


def refine_values(dw, x, offsets, cols) -> np.ndarray:
    """Least-squares values on the chosen columns against the layer output error."""
    dw = np.asarray(dw, dtype=np.float64)
    x = np.asarray(x, dtype=np.float64)
    rows, n = dw.shape
    basis = sylvester(n) / np.sqrt(n)
    out = np.empty(int(offsets[-1]))
    for r in range(rows):
        sel = cols[offsets[r]:offsets[r + 1]]
        if sel.size == 0:
            continue
        a = (basis[sel, :] @ x).T              # [T, k_r]
        b = dw[r] @ x                           # [T]
        out[offsets[r]:offsets[r + 1]] = np.linalg.lstsq(a, b, rcond=None)[0]
    return out


def to_fixed_width(offsets, cols, values):
    """[rows, k_max] values and columns; short rows padded with zero values on their first column."""
    counts = np.diff(offsets)
    rows, kmax = counts.size, int(counts.max(initial=0))
    v = np.zeros((rows, kmax), dtype=np.float64)
    c = np.zeros((rows, kmax), dtype=np.int32)
    for r in range(rows):
        k = int(counts[r])
        if k == 0:
            continue
        c[r, :k] = cols[offsets[r]:offsets[r + 1]]
        c[r, k:] = c[r, 0]
        v[r, :k] = values[offsets[r]:offsets[r + 1]]
    return v, c


def expand_two_sided(values, cols, m: int, n: int) -> np.ndarray:
    """dense[b] = (H_m / sqrt m) scatter(values, cols)[b] (H_n / sqrt n); values, cols [batch, m, nnz]."""
    f = scatter_dense(values, cols, n)
    if f.shape[1] != m:
        raise ValueError("values must have m rows per batch")
    return (sylvester(m) / np.sqrt(m)) @ f @ (sylvester(n) / np.sqrt(n))


def gather_two_sided(grad, cols) -> np.ndarray:
    """The adjoint of expand_two_sided: ((H_m / sqrt m) G (H_n / sqrt n))[b, r, cols[b, r, k]]."""
    g = np.asarray(grad, dtype=np.float64)
    m, n = g.shape[-2:]
    full = (sylvester(m) / np.sqrt(m)) @ g @ (sylvester(n) / np.sqrt(n))
    return np.take_along_axis(full, np.asarray(cols, dtype=np.int64), axis=-1)
