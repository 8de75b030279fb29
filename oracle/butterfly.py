"""Mixed-radix stride butterfly rotation, in float64 (test oracle only).

HARP explainer, technical summary §2.1: for a length d and a mixed-radix
schedule b = (b_0, ..., b_{m-1}) with prod b_t = d, stage t applies a
block-diagonal orthogonal matrix B_t to groups of coordinates separated by a
stride permutation; §2.2: each block B_{t,c} is b_t x b_t, and with all blocks
equal to the normalized Sylvester Hadamard H_b / sqrt(b) the product recovers
the fixed Hadamard transform up to a fixed permutation convention.

Convention chosen (the pages leave it open):

* index i = sum_t i_t * S_t with S_t = prod_{u > t} b_u (row-major digits,
  digit 0 most significant);
* stage t maps x[i] <- sum_k B_{t,c}[i_t, k] * x[i with digit t set to k],
  where the group id c enumerates the other digits in row-major order with
  digit t removed;
* stages apply t = 0 first, so R = B_{m-1} ... B_0; R^T applies the transposed
  blocks in reverse order;
* a stage may carry one block per group (d / b_t blocks) or one block shared
  by every group.

With every block equal to H_b / sqrt(b) this convention gives exactly
H_d / sqrt(d) because the Sylvester matrices satisfy H_a (x) H_b = H_ab.

The randomized transform for lengths that are not powers of two (HARP
explainer, technical summary §2.1: stride stages for any factorization of d,
e.g. d = 5120 = 8 * 8 * 8 * 5 * 2) is read the same way as the power-of-two
RHT: y = R diag(s) x, with Hadamard blocks H_b / sqrt(b) for the power-of-two
radices and orthogonal mixers for the others; its inverse is
x = diag(s) R^T y.

Pinned by tests/test_oracle_butterfly.py: a pure-Python index-loop evaluation
of the definition on tiny schedules, the all-Hadamard case against the
popcount formula for H_d, a single full-width stage against a dense matrix
product, orthogonality of the dense R, and R^T R = I; the mixed-radix RHT
against the dense Sylvester RHT when every radix is a power of two, norm
preservation with a radix-5 mixer, and inverse after forward.
"""
from __future__ import annotations

import numpy as np

from .hadamard import is_pow2, sylvester


def strides(radices) -> list[int]:
    out, acc = [], 1
    for b in reversed(radices):
        out.append(acc)
        acc *= int(b)
    return list(reversed(out))


def apply_stages(x, radices, blocks, transpose: bool = False) -> np.ndarray:
    """Apply R (or R^T) to every row of x.

    x: [rows, d]; radices: (b_0, ..., b_{m-1}); blocks[t]: [G_t, b_t, b_t] with
    G_t = d / b_t (one block per group) or G_t = 1 (shared by all groups).
    """
    x = np.asarray(x, dtype=np.float64)
    rows, d = x.shape
    radices = [int(b) for b in radices]
    if int(np.prod(radices)) != d:
        raise ValueError("radices must multiply to d")
    xt = x.reshape(rows, *radices)
    order = range(len(radices)) if not transpose else reversed(range(len(radices)))
    for t in order:
        b = radices[t]
        blk = np.asarray(blocks[t], dtype=np.float64)
        if blk.shape[-2:] != (b, b) or blk.shape[0] not in (1, d // b):
            raise ValueError(f"stage {t}: blocks must be [d/b or 1, b, b]")
        if transpose:
            blk = np.swapaxes(blk, -1, -2)
        moved = np.moveaxis(xt, 1 + t, -1)          # [rows, other digits..., b]
        others = moved.shape[1:-1]
        if blk.shape[0] == 1:
            bt = np.broadcast_to(blk[0], (*others, b, b))
        else:
            bt = blk.reshape(*others, b, b)         # group c = other digits, row-major
        out = np.einsum("r...k,...ik->r...i", moved, bt)
        xt = np.moveaxis(out, -1, 1 + t)
    return np.ascontiguousarray(xt).reshape(rows, d)


def apply_stages_cols(x, radices, blocks, transpose: bool = False) -> np.ndarray:
    """Apply R (or R^T) to every column of x (transform length = rows)."""
    return apply_stages(np.asarray(x, dtype=np.float64).T, radices, blocks, transpose).T


def dense(radices, blocks, transpose: bool = False) -> np.ndarray:
    """The dense d x d matrix R (or R^T): column j is R e_j."""
    d = int(np.prod(radices))
    return apply_stages(np.eye(d), radices, blocks, transpose).T


def two_sided(w, radices_in, blocks_in, radices_out, blocks_out) -> np.ndarray:
    """W' = R_out W R_in^T: R_in along every row, R_out along every column."""
    return apply_stages_cols(apply_stages(w, radices_in, blocks_in), radices_out, blocks_out)


def rht_stage_blocks(radices, mixers=None) -> list[np.ndarray]:
    """Stage blocks of the mixed-radix RHT: the shared [1, b, b] block H_b / sqrt(b)
    for a power-of-two radix, the given orthogonal blocks mixers[b] otherwise."""
    out = []
    for b in (int(v) for v in radices):
        if is_pow2(b):
            out.append((sylvester(b) / np.sqrt(b))[None])
        elif mixers is None or b not in mixers:
            raise ValueError(f"radix {b} is not a power of two: its orthogonal blocks must be given")
        else:
            out.append(np.asarray(mixers[b], dtype=np.float64))
    return out


def rht_mixed(x, signs, radices, blocks) -> np.ndarray:
    """y = R diag(s) x for every row of x (signs applied first)."""
    x = np.asarray(x, dtype=np.float64) * np.asarray(signs, dtype=np.float64)
    return apply_stages(x, radices, blocks)


def irht_mixed(y, signs, radices, blocks) -> np.ndarray:
    """x = diag(s) R^T y for every row of y (the inverse of rht_mixed)."""
    return apply_stages(y, radices, blocks, transpose=True) * np.asarray(signs, dtype=np.float64)
