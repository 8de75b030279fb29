"""The quantizer's arithmetic, isolated from transform rounding.

When every partial sum of the fast WHT is an integer (or a fixed multiple of a
power of two) below 2^24, the fp32 transform on the GPU is exact, so the GPU
quantizes exactly the values the oracle quantizes.  Its codes must then equal
the oracle's codes bit for bit -- no rounding-boundary window is excused --
and its scales must be equal, which checks the correctly rounded division
(t = RN(y / s)), the ties-to-even rounding and the packing on their own.

Inputs are built from chosen transform outputs y: for a row of n = 2^k with k
even, x = D H y / sqrt(n) is exact when |H y| < 2^24, and H D x = n y is then
computed exactly too (after j stages the partial sums are 2^j times the WHT of
y over the remaining bits, bounded by n max|y|).  Choosing y near
(k + 1/2) s, with s = RN(max|y| / qmax), puts many quotients within an ulp of a
rounding boundary.
"""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
from oracle import hadamard as oh
from oracle import quant as oq
from tests._parity import to_gpu_bf16, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu


def exact_input_for(y: np.ndarray, signs: np.ndarray) -> np.ndarray:
    """x with rht(x) == y exactly (y integer-valued times a power of two)."""
    n = y.shape[1]
    x = oh.irht_rows(y.astype(np.float64), signs)  # D H y / sqrt(n), exact in float64
    xf = x.astype(np.float32)
    assert np.array_equal(xf.astype(np.float64), x), "input not exactly representable"
    return xf


def near_tie_rows(rng, rows: int, n: int, group: int, bits: int, lim: int) -> np.ndarray:
    """Integer rows whose quotients y/s sit on or next to half-integers."""
    qm = np.float32((1 << (bits - 1)) - 1)
    y = np.zeros((rows, n), np.float64)
    for r in range(rows):
        for g0 in range(0, n, group):
            A = int(rng.integers(lim // 2, lim))
            if r % 4 == 0:  # exact ties: s a power of two
                A = int(qm) * (1 << int(rng.integers(4, max(5, int(np.log2(lim / qm))))))
            s = float(np.float32(np.float32(A) / qm))
            k = rng.integers(-int(qm), int(qm), size=group).astype(np.float64)
            v = np.rint((k + 0.5) * s + rng.integers(-1, 2, size=group))
            v = np.clip(v, -A, A)
            v[int(rng.integers(group))] = A * (1 if rng.random() < 0.5 else -1)
            y[r, g0:g0 + group] = v
    return y


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("scale_pow", [0, -135, 100])
def test_near_ties_bit_exact(bits, group, scale_pow):
    """n = 64 rows (one thread per row) built so that many y/s are within an
    ulp of k + 1/2, including exact ties; scale_pow moves the whole problem to
    subnormal or huge scales (exact power-of-two rescaling on both sides)."""
    n = 64
    rng = np.random.default_rng(1000 * bits + group + scale_pow)
    y = near_tie_rows(rng, 2000, n, group, bits, lim=1 << 17) * 2.0 ** scale_pow
    signs = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    x = exact_input_for(y, signs)
    codes, scales = hit.rht_quantize_pack(to_gpu_f32(x), to_gpu_i8(signs), bits, group)
    torch.cuda.synchronize()
    ref = oq.quantize(y, bits, group)
    u = oq.unpack(codes.cpu().numpy(), bits, n)
    bad = int((u != ref["u"]).sum())
    near = int(oq.boundary_window(ref["t"]).sum())
    assert near > 100, "the construction should put many quotients near a boundary"
    assert bad == 0, f"{bad} codes differ (of {u.size}, {near} near a boundary)"
    assert np.array_equal(scales.cpu().numpy(), ref["scales"])


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_stream_kernel_integer_rows_bit_exact(bits, dtype):
    """n = 4096 through the persistent row kernel: integer inputs (|x| < 2^12,
    or < 2^8 for bf16) make every partial sum an integer below 2^24, so the
    transform is exact and all 24-bit quotients must quantize exactly."""
    n, rows = 4096, 1500
    rng = np.random.default_rng(77 + bits)
    lim = 4096 if dtype == "f32" else 256
    x = rng.integers(-lim + 1, lim, size=(rows, n)).astype(np.float32)
    x[7] = 0.0
    signs = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    if dtype == "f32":
        xg = to_gpu_f32(x)
    else:
        bits16 = (x.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal((bits16.astype(np.uint32) << 16).view(np.float32), x)
        xg = to_gpu_bf16(bits16)
    for group in (64, 128, 4096):
        codes, scales = hit.rht_quantize_pack(xg, to_gpu_i8(signs), bits, group)
        torch.cuda.synchronize()
        ref = oq.quantize(oh.rht_rows(x.astype(np.float64), signs), bits, group)
        u = oq.unpack(codes.cpu().numpy(), bits, n)
        assert int((u != ref["u"]).sum()) == 0
        assert np.array_equal(scales.cpu().numpy(), ref["scales"])
