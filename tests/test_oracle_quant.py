"""Pins for the oracle's group quantizer, packing and dequantization (CPU only).

The fp32 rounding of every step is re-derived with exact rational arithmetic
(fractions.Fraction), independently of numpy's float32 division.
"""
from fractions import Fraction

import numpy as np
import pytest

from oracle import quant as oq
from tests._golden import quant_cases


def rn_f32(x: Fraction) -> Fraction:
    """Round a rational to the nearest IEEE binary32 value, ties to even."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    ulp = Fraction(2) ** (e - 23)
    m = round(a / ulp)              # Python rounds Fractions half to even
    return sign * m * ulp


def exact_group(y, bits):
    qmax = (1 << (bits - 1)) - 1
    ys = [Fraction(float(v)) for v in y]
    a = max(abs(v) for v in ys)
    s = rn_f32(a / qmax)
    if s == 0:
        return s, [Fraction(0)] * len(ys), [0] * len(ys)
    t = [rn_f32(v / s) for v in ys]
    q = [max(-qmax, min(qmax, round(v))) for v in t]
    return s, t, q


@pytest.mark.parametrize("case", list(quant_cases()), ids=lambda c: f"b{c[0]}")
def test_hand_worked_examples(case):
    bits, y, scale, q, packed, yhat = case
    r = oq.quantize(y[None, :], bits, 4)
    assert r["scales"][0, 0] == scale
    assert np.array_equal(r["q"][0], q)
    codes = oq.pack(r["u"], bits)
    assert bytes(codes[0]) == packed
    assert np.array_equal(oq.unpack(codes, bits, 4), r["u"])
    deq = oq.dequantize(r["u"], r["scales"], bits, 4)
    assert np.array_equal(deq[0], yhat)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_every_rounding_step_matches_exact_rationals(bits):
    rng = np.random.default_rng(100 + bits)
    g = 16
    y = (rng.standard_normal((6, 4 * g)) * 0.02).astype(np.float32)
    y[0, 3] *= 50
    y[1, :g] = 0.0                      # an all-zero group
    y[2, g:2 * g] = np.float32(1e-39)   # subnormal inputs
    y[3, 5] = np.float32(-3.0e38)       # huge magnitude
    r = oq.quantize(y, bits, g)
    for row in range(y.shape[0]):
        for grp in range(4):
            seg = y[row, grp * g:(grp + 1) * g]
            s, t, q = exact_group(seg, bits)
            assert Fraction(float(r["scales"][row, grp])) == s
            got_t = [Fraction(float(v)) for v in r["t"][row, grp * g:(grp + 1) * g]]
            assert got_t == t
            assert list(r["q"][row, grp * g:(grp + 1) * g]) == q


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_invariants(bits):
    rng = np.random.default_rng(bits)
    y = rng.standard_t(3, size=(32, 256)).astype(np.float32)
    r = oq.quantize(y, bits, 64)
    qmax = (1 << (bits - 1)) - 1
    g = np.abs(y).reshape(32, 4, 64)
    arg = np.argmax(g, axis=-1)
    qg = r["q"].reshape(32, 4, 64)
    picked = np.take_along_axis(qg, arg[..., None], axis=-1)[..., 0]
    assert np.all(np.abs(picked) == qmax)
    deq = oq.dequantize(r["u"], r["scales"], bits, 64)
    s = np.repeat(r["scales"], 64, axis=1).astype(np.float64)
    err = np.abs(deq.astype(np.float64) - y.astype(np.float64))
    assert np.all(err <= s / 2 * (1 + 1e-6) + 1e-30)
    assert r["u"].min() >= 1 and r["u"].max() <= 2 * qmax + 1


def test_pack_layout_by_hand():
    # 4-bit: low nibble holds the even element
    assert bytes(oq.pack(np.array([[1, 2, 3, 4]], np.uint8), 4)[0]) == bytes([0x21, 0x43])
    # 2-bit: element j at bits 2j..2j+1
    assert bytes(oq.pack(np.array([[0, 1, 2, 3]], np.uint8), 2)[0]) == bytes([0b11100100])
    # 3-bit: eight codes fill three bytes: 0..7 -> stream sum(j << 3j)
    stream = sum(j << (3 * j) for j in range(8))
    assert bytes(oq.pack(np.arange(8, dtype=np.uint8)[None, :], 3)[0]) == stream.to_bytes(3, "little")


@pytest.mark.parametrize("bits,n", [(2, 64), (3, 64), (4, 64), (3, 8192)])
def test_pack_unpack_round_trip(bits, n):
    rng = np.random.default_rng(n + bits)
    u = rng.integers(0, 1 << bits, size=(3, n), dtype=np.uint8)
    c = oq.pack(u, bits)
    assert c.shape == (3, n * bits // 8)
    assert np.array_equal(oq.unpack(c, bits, n), u)


def test_boundary_window():
    t = np.array([0.5, 0.5 + 2e-6, 0.5 + 5e-7, 6.5 - 6e-6, 6.5 - 7e-6, -2.5, 3.0], np.float32)
    w = oq.boundary_window(t)
    assert list(w) == [True, False, True, True, False, True, False]


def test_rejects_bad_arguments():
    with pytest.raises(ValueError):
        oq.quantize(np.zeros((1, 8), np.float32), 5, 4)
    with pytest.raises(ValueError):
        oq.quantize(np.zeros((1, 8), np.float32), 4, 3)
