"""Group-wise symmetric absmax round-to-nearest quantizer, code packing and
dequantization, in scalar fp32 (test oracle only).

The pages name a "blockwise" scalar quantizer as the backend that consumes the
rotated weights (HARP explainer, technical summary §1 and §2.3) but fix no
format.  The workloads fix symmetric absmax RTN with 2/3/4-bit codes in groups
of contiguous elements along a row; the remaining choices are readings:

* qmax = 2^(b-1) - 1 (symmetric: 4-bit uses -7..7, 3-bit -3..3, 2-bit -1..1);
* every step in IEEE fp32: yf = fp32(y), a = max |yf| over the group,
  s = a / qmax (correctly rounded division), t = yf / s (correctly rounded),
  q = clamp(rint(t), -qmax, qmax) with ties to even; a = 0 gives s = 0 and q = 0;
* stored code u = q + 2^(b-1) (offset binary), packed least-significant bit
  first into a per-row bit stream: code j occupies stream bits [b*j, b*j + b)
  and stream bit k is bit (k mod 8) of byte k // 8.  For b = 4 this is two
  codes per byte (low nibble first), for b = 2 four per byte, for b = 3 eight
  codes per three bytes;
* scales are fp32, row-major [rows, n / group];
* dequantized value yhat = fp32(q) * s (one fp32 multiply).

Pinned by tests/test_oracle_quant.py: hand-worked group-of-4 examples
(tests/golden/quant_hand_examples.txt), an exact rational re-derivation of each
fp32 rounding step on random groups, tie cases, the invariants (the absmax
element maps to +-qmax, |y - yhat| <= s/2, zero groups), and pack/unpack
round trips against hand-written bit streams.
"""
from __future__ import annotations

import numpy as np


def qmax_of(bits: int) -> int:
    if bits not in (2, 3, 4):
        raise ValueError("bits must be 2, 3 or 4")
    return (1 << (bits - 1)) - 1


def quantize(y, bits: int, group: int) -> dict:
    """Quantize each row of y (any float array, rounded once to fp32) in groups.

    Returns dict with q (int8 codes -qmax..qmax), u (uint8 stored codes),
    scales (fp32 [rows, n/group]), t (fp32 pre-rounding values in code units)
    and yf (the fp32 values that were quantized).
    """
    yf = np.asarray(y).astype(np.float32)
    if yf.ndim != 2:
        raise ValueError("y must be 2-D [rows, n]")
    rows, n = yf.shape
    if group <= 0 or n % group:
        raise ValueError("group must divide n")
    qm = np.float32(qmax_of(bits))
    g = yf.reshape(rows, n // group, group)
    a = np.max(np.abs(g), axis=-1) if n else np.zeros((rows, 0), np.float32)
    s = (a / qm).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    t = (g / safe[..., None]).astype(np.float32)
    t = np.where(s[..., None] > 0, t, np.float32(0.0)).astype(np.float32)
    q = np.clip(np.rint(t), -qm, qm).astype(np.int8)
    u = (q.astype(np.int16) + (1 << (bits - 1))).astype(np.uint8)
    return {"q": q.reshape(rows, n), "u": u.reshape(rows, n), "scales": s,
            "t": t.reshape(rows, n), "yf": yf}


def pack(u, bits: int) -> np.ndarray:
    """Pack stored codes [rows, n] into the LSB-first bit stream
    [rows, ceil(n*bits/8)]; a row's last byte is padded with zero bits."""
    u = np.asarray(u, dtype=np.uint8)
    rows, n = u.shape
    stream = ((u[..., None] >> np.arange(bits, dtype=np.uint8)) & 1).astype(np.uint8)
    return np.packbits(stream.reshape(rows, n * bits), axis=-1, bitorder="little")


def unpack(codes, bits: int, n: int) -> np.ndarray:
    """Inverse of :func:`pack`: stored codes [rows, n] from packed bytes."""
    codes = np.asarray(codes, dtype=np.uint8)
    rows = codes.shape[0]
    stream = np.unpackbits(codes, axis=-1, bitorder="little")[:, : n * bits]
    stream = stream.reshape(rows, n, bits).astype(np.uint8)
    return (stream << np.arange(bits, dtype=np.uint8)).sum(axis=-1).astype(np.uint8)


def dequantize(u, scales, bits: int, group: int) -> np.ndarray:
    """yhat = fp32(u - 2^(b-1)) * s, one fp32 multiply per element."""
    u = np.asarray(u, dtype=np.uint8)
    rows, n = u.shape
    q = (u.astype(np.int16) - (1 << (bits - 1))).astype(np.float32)
    s = np.asarray(scales, dtype=np.float32).reshape(rows, n // group)
    yhat = q.reshape(rows, n // group, group) * s[..., None]
    return yhat.astype(np.float32).reshape(rows, n)


def boundary_window(t, tol: float = 1e-6) -> np.ndarray:
    """Elements whose pre-rounding value t lies within tol * max(1, |k + 1/2|) of a
    rounding boundary k + 1/2 (evaluated in float64 on the fp32 t)."""
    t64 = np.asarray(t, dtype=np.float64)
    k_half = np.floor(t64) + 0.5
    return np.abs(t64 - k_half) <= tol * np.maximum(1.0, np.abs(k_half))
