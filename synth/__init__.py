"""Seeded synthetic inputs for the five Hadamard-incoherence workloads.

This module is shared by the CPU oracle and the CUDA path, so it holds no
arithmetic of the method itself: it only draws random numbers (values,
outlier positions, sign vectors, orthogonal blocks, sparse index lists) and
converts them to the storage types the workloads name.  Every generator takes
its shape as arguments so tests can draw small versions of the same recipe;
the defaults are the full workload sizes.

Recipes (one seed per workload, child streams per quantity):

* ``weight_rht_int4``   fp32 [4096, 4096] ~ N(0, 0.02^2); 0.1 % of entries
  (rounded) at distinct seeded positions multiplied by 50; Rademacher signs.
* ``activation_rht``    bf16 [8192, 4096] = 0.5 * Student-t(nu=3); 1 % of
  columns (rounded) multiplied by 20; rounded to bf16 (nearest-even).
* ``two_sided_butterfly`` bf16 [4096, 14336] ~ N(0, 0.02^2); per-stage
  block-diagonal orthogonal blocks (QR of a seeded Gaussian, sign-fixed) for
  radices (7, 16, 16, 8) along rows and (16, 16, 16) along columns.
* ``two_sided_lowbit``  bf16 [8192, 8192] ~ N(0, 0.02^2); 0.05 % of entries
  multiplied by 100; row and column Rademacher signs.
* ``wht_adapter``       [32, 4096, 64] fp32 values ~ N(0, (1e-3)^2) and int32
  column indices: 64 distinct uniform columns per row, sorted ascending.
* ``mixed_rht_int4``    fp32 [4096, 5120] as the weight recipe; radices
  (8, 8, 8, 5, 2): one seeded orthogonal 5 x 5 mixer shared by every group
  (the power-of-two radices use Hadamard blocks, which are not inputs).
* ``harp_rotation``     fp32 [4096, d] as the weight recipe; Rademacher signs;
  per stage and group the learnable parameters ~ N(0, 0.05^2) (a small
  refinement around the zero start); d = 4096 with radices (16, 16, 16), or
  d = 5120 with (8, 8, 8, 5, 2) and one seeded orthogonal mixer for radix 5.
* ``qwha_init``         fp32 weight [4096, 4096] as the weight recipe with
  Rademacher signs (its quantization error is what the adapter targets);
  activations fp32 [4096, 512] ~ N(0, 1) with 1 % of input channels (rounded)
  multiplied by 20; a budget of 64 parameters per row on average with at
  least 1 per row.
"""
from __future__ import annotations

import numpy as np

BASE_SEED = 20260

WORKLOADS = {
    "weight_rht_int4": 1,
    "activation_rht": 2,
    "two_sided_butterfly": 3,
    "two_sided_lowbit": 4,
    "wht_adapter": 5,
    "mixed_rht_int4": 6,
    "harp_rotation": 7,
    "qwha_init": 8,
}


def streams(workload: str, k: int, seed: int | None = None):
    """k independent numpy Generators for one workload (PCG64 child streams)."""
    s = BASE_SEED + WORKLOADS[workload] if seed is None else seed
    return [np.random.Generator(np.random.PCG64(c)) for c in np.random.SeedSequence(s).spawn(k)]


def rademacher(rng: np.random.Generator, n: int) -> np.ndarray:
    """i.i.d. +-1 signs as int8."""
    return (rng.integers(0, 2, size=n, dtype=np.int8) * 2 - 1).astype(np.int8)


def distinct_positions(rng: np.random.Generator, population: int, count: int) -> np.ndarray:
    """`count` distinct integers drawn uniformly from [0, population), sorted."""
    if count > population:
        raise ValueError("count exceeds population")
    got = np.unique(rng.integers(0, population, size=count, dtype=np.int64))
    while got.size < count:
        extra = rng.integers(0, population, size=count - got.size, dtype=np.int64)
        got = np.unique(np.concatenate([got, extra]))
    return got


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the raw uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def seeded_orthogonal_blocks(rng: np.random.Generator, count: int, b: int) -> np.ndarray:
    """`count` random b x b orthogonal matrices: QR of a Gaussian, Q * sign(diag R)."""
    a = rng.standard_normal((count, b, b))
    q, r = np.linalg.qr(a)
    d = np.sign(np.diagonal(r, axis1=-2, axis2=-1))
    d[d == 0] = 1.0
    return (q * d[:, None, :]).astype(np.float32)


def weight_rht_int4(rows: int = 4096, n: int = 4096, seed: int | None = None) -> dict:
    rv, rp, rs = streams("weight_rht_int4", 3, seed)
    x = (rv.standard_normal((rows, n)) * 0.02).astype(np.float32)
    cnt = int(round(0.001 * rows * n))
    pos = distinct_positions(rp, rows * n, cnt)
    x.reshape(-1)[pos] *= np.float32(50.0)
    return {"x": x, "signs": rademacher(rs, n), "bits": 4, "group": 128, "outliers": pos}


def activation_rht(rows: int = 8192, n: int = 4096, seed: int | None = None) -> dict:
    rv, rc, rs = streams("activation_rht", 3, seed)
    x = (0.5 * rv.standard_t(3.0, size=(rows, n))).astype(np.float32)
    cols = distinct_positions(rc, n, int(round(0.01 * n)))
    x[:, cols] *= np.float32(20.0)
    return {"x_bf16": to_bf16_bits(x), "signs": rademacher(rs, n), "outlier_cols": cols}


def two_sided_butterfly(rows: int = 4096, d: int = 14336,
                        radices_in=(7, 16, 16, 8), radices_out=(16, 16, 16),
                        seed: int | None = None) -> dict:
    if int(np.prod(radices_in)) != d or int(np.prod(radices_out)) != rows:
        raise ValueError("radices must multiply to the transformed length")
    rv, rbi, rbo = streams("two_sided_butterfly", 3, seed)
    x = (rv.standard_normal((rows, d)) * 0.02).astype(np.float32)
    blocks_in = [seeded_orthogonal_blocks(rbi, d // b, b) for b in radices_in]
    blocks_out = [seeded_orthogonal_blocks(rbo, rows // b, b) for b in radices_out]
    return {"x_bf16": to_bf16_bits(x), "radices_in": tuple(radices_in), "blocks_in": blocks_in,
            "radices_out": tuple(radices_out), "blocks_out": blocks_out}


def mixed_rht_int4(rows: int = 4096, d: int = 5120, radices=(8, 8, 8, 5, 2), seed: int | None = None) -> dict:
    """Rows of length d = prod(radices) (not a power of two), N(0, 0.02) with
    0.1 % outliers x 50; Rademacher signs; for every radix b that is not a power
    of two, one seeded orthogonal mixer shared by all groups ([1, b, b] under
    key b).  The power-of-two radices carry no input: their blocks are the
    Hadamard ones."""
    if int(np.prod(radices)) != d:
        raise ValueError("radices must multiply to d")
    rv, rp, rs, rb = streams("mixed_rht_int4", 4, seed)
    x = (rv.standard_normal((rows, d)) * 0.02).astype(np.float32)
    pos = distinct_positions(rp, rows * d, int(round(0.001 * rows * d)))
    x.reshape(-1)[pos] *= np.float32(50.0)
    mixers = {b: seeded_orthogonal_blocks(rb, 1, b) for b in sorted(set(radices)) if b & (b - 1)}
    return {"x": x, "signs": rademacher(rs, d), "radices": tuple(radices), "mixers": mixers, "bits": 4,
            "group": 128}


def harp_rotation(rows: int = 4096, d: int = 4096, radices=(16, 16, 16), theta_std: float = 0.05,
                  seed: int | None = None) -> dict:
    """Weights, signs and per-stage learnable parameters [d / b_t, P(b_t)] with
    P(1) = 0, P(2) = 1 and P(b) = b (b - 1) / 2; one seeded orthogonal mixer per
    radix that is not a power of two."""
    radices = tuple(int(b) for b in radices)
    if int(np.prod(radices)) != d:
        raise ValueError("radices must multiply to d")
    rv, rp, rs, rt, rm = streams("harp_rotation", 5, seed)
    x = (rv.standard_normal((rows, d)) * 0.02).astype(np.float32)
    pos = distinct_positions(rp, rows * d, int(round(0.001 * rows * d)))
    x.reshape(-1)[pos] *= np.float32(50.0)
    counts = [0 if b == 1 else 1 if b == 2 else b * (b - 1) // 2 for b in radices]
    thetas = [(rt.standard_normal((d // b, p)) * theta_std).astype(np.float32) for b, p in zip(radices, counts)]
    base = {b: seeded_orthogonal_blocks(rm, 1, b)[0] for b in sorted(set(radices)) if b & (b - 1)}
    return {"x": x, "signs": rademacher(rs, d), "radices": radices, "thetas": thetas, "base_mixers": base,
            "bits": 4, "group": 128}


def qwha_init(rows: int = 4096, n: int = 4096, tokens: int = 512, per_row: int = 64, k_min: int = 1,
              seed: int | None = None) -> dict:
    """Weights to be quantized, Rademacher signs for the rotated quantizer,
    synthetic activations with outlier input channels, and the parameter budget."""
    rv, rp, rs, rx, rc = streams("qwha_init", 5, seed)
    w = (rv.standard_normal((rows, n)) * 0.02).astype(np.float32)
    pos = distinct_positions(rp, rows * n, int(round(0.001 * rows * n)))
    w.reshape(-1)[pos] *= np.float32(50.0)
    x = rx.standard_normal((n, tokens)).astype(np.float32)
    hot = distinct_positions(rc, n, int(round(0.01 * n)))
    x[hot, :] *= np.float32(20.0)
    return {"w": w, "signs": rademacher(rs, n), "x": x, "budget": per_row * rows, "k_min": k_min,
            "bits": 4, "group": 128, "outlier_channels": hot}


def two_sided_lowbit(rows: int = 8192, n: int = 8192, seed: int | None = None) -> dict:
    rv, rp, rs, rc = streams("two_sided_lowbit", 4, seed)
    x = (rv.standard_normal((rows, n)) * 0.02).astype(np.float32)
    cnt = int(round(0.0005 * rows * n))
    pos = distinct_positions(rp, rows * n, cnt)
    x.reshape(-1)[pos] *= np.float32(100.0)
    return {"x_bf16": to_bf16_bits(x), "row_signs": rademacher(rs, n),
            "col_signs": rademacher(rc, rows), "group": 64, "outliers": pos}


def sparse_columns(rng: np.random.Generator, rows: int, n: int, nnz: int) -> np.ndarray:
    """For each row, `nnz` distinct columns drawn uniformly from [0, n), sorted (int32)."""
    if nnz > n:
        raise ValueError("nnz exceeds n")
    cols = np.sort(rng.integers(0, n, size=(rows, nnz), dtype=np.int64), axis=1)
    while True:
        dup = np.zeros_like(cols, dtype=bool)
        dup[:, 1:] = cols[:, 1:] == cols[:, :-1]
        k = int(dup.sum())
        if k == 0:
            return cols.astype(np.int32)
        cols[dup] = rng.integers(0, n, size=k, dtype=np.int64)
        cols.sort(axis=1)


def wht_adapter(batch: int = 32, rows: int = 4096, n: int = 4096, nnz: int = 64,
                seed: int | None = None) -> dict:
    rv, rc, rg = streams("wht_adapter", 3, seed)
    values = (rv.standard_normal((batch, rows, nnz)) * 1e-3).astype(np.float32)
    cols = sparse_columns(rc, batch * rows, n, nnz).reshape(batch, rows, nnz)
    return {"values": values, "cols": cols, "n": n}


def dense_gradient(batch: int, rows: int, n: int, seed: int | None = None) -> np.ndarray:
    """A seeded dense upstream gradient for the adapter backward, N(0, 1)."""
    s = BASE_SEED + 1000 + WORKLOADS["wht_adapter"] if seed is None else seed
    rg = np.random.Generator(np.random.PCG64(s))
    return rg.standard_normal((batch, rows, n)).astype(np.float32)
