"""GPU parity of the QWHA pieces around the sparse expansion (through the C
ABI): the two-transform expansion and its gradient, row norms, the per-row
top-k selection, and the AdaAlloc initialisation pipeline on the synthetic
recipe, against oracle.qwha."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import hadamard as oh
from oracle import quant as oq
from oracle import qwha as oqw
from tests._parity import assert_close, host, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu


def sparse(batch, m, n, nnz, seed, dup=False):
    rng = np.random.default_rng(seed)
    vals = (rng.standard_normal((batch, m, nnz)) * 1e-3).astype(np.float32)
    cols = np.stack([np.stack([rng.choice(n, nnz, replace=False) for _ in range(m)]) for _ in range(batch)])
    cols = cols.astype(np.int32)
    if dup:
        cols[:, :, 1] = cols[:, :, 0]  # duplicates add up
    return vals, cols


@pytest.mark.parametrize("batch,m,n,nnz", [(2, 256, 1024, 16), (1, 2048, 512, 7), (2, 4096, 4096, 64)])
def test_two_sided_expansion_and_gradient(batch, m, n, nnz):
    vals, cols = sparse(batch, m, n, nnz, m + n, dup=(m == 256))
    dense = hit.wht_expand_2d(to_gpu_f32(vals), torch.from_numpy(cols).cuda(), n, 1 / np.sqrt(n))
    torch.cuda.synchronize()
    ref = oqw.expand_two_sided(vals, cols, m, n)
    assert_close(host(dense), ref, torch.float32, "two-sided expansion")
    g = np.random.default_rng(1).standard_normal((batch, m, n)).astype(np.float32)
    gd = to_gpu_f32(g)
    grad = hit.wht_gather_2d(gd, torch.from_numpy(cols).cuda(), 1 / np.sqrt(n))
    torch.cuda.synchronize()
    assert np.array_equal(gd.cpu().numpy(), g), "the incoming gradient must not be modified"
    assert_close(host(grad), oqw.gather_two_sided(g, cols), torch.float32, "two-sided gradient")


def test_row_norms():
    x = np.random.default_rng(3).standard_normal((333, 4096)).astype(np.float32)
    x[5] = 0.0
    got = hit.row_norms(to_gpu_f32(x)).cpu().numpy()
    want = oqw.channel_error(x.astype(np.float64))
    assert np.allclose(got, want, rtol=1e-12, atol=0.0)


@pytest.mark.parametrize("n", [1024, 4096, 8192])
def test_select_equals_oracle_with_ties(n):
    rng = np.random.default_rng(n)
    rows = 97
    f = (rng.standard_normal((rows, n)) * 1e-3).astype(np.float32)
    f[::3] = np.round(f[::3] * 4e3) / 4e3           # many exact ties in magnitude
    f[1::5, :200] = 0.0
    f[2, :] = 1.0                                     # one row entirely tied
    counts = rng.integers(0, n + 1, size=rows)
    counts[:6] = (0, 1, n, n - 1, 5, 64)
    off = np.zeros(rows + 1, np.int64)
    off[1:] = np.cumsum(counts)
    cols, vals = hit.qwha_select(to_gpu_f32(f), torch.from_numpy(off).cuda())
    torch.cuda.synchronize()
    woff, wcols = oqw.select(f.astype(np.float64), counts)
    assert np.array_equal(cols.cpu().numpy(), wcols)
    assert np.array_equal(vals.cpu().numpy(), oqw.direct_values(f.astype(np.float64), woff, wcols).astype(np.float32))


def test_adaalloc_initialisation_pipeline():
    """On the synthetic recipe (4096 x 4096 weights, budget 64 per row, at
    least 1): the rotated quantizer's error dW on the device, its coefficients
    F* = dW H / sqrt(n), the channel errors, the budget split and the per-row
    selection.  Each device stage is compared with the oracle applied to the
    device's previous stage (codes are compared with the oracle's in the
    quantizer tests; an excused boundary code would otherwise dominate the
    residual): the reconstruction of the codes and the coefficients within the
    fp32 tolerance, the errors within 1e-12, and the split and the selection
    bit for bit."""
    d = synth.qwha_init()
    rows, n = d["w"].shape
    w = to_gpu_f32(d["w"])
    s = to_gpu_i8(d["signs"])
    codes, scales = hit.rht_quantize_pack(w, s, d["bits"], d["group"])
    w_hat = hit.dequant_inverse(codes, scales, n, d["bits"], d["group"], s)
    dw = w - w_hat                                   # test-side residual of two library outputs
    coef = hit.rht_forward(dw)                       # F* = dW H / sqrt(n) (no signs)
    err = hit.row_norms(dw)
    torch.cuda.synchronize()
    u = oq.unpack(codes.cpu().numpy(), d["bits"], n)
    w_hat_ref = oh.irht_rows(oq.dequantize(u, scales.cpu().numpy(), d["bits"], d["group"]), d["signs"])
    assert_close(host(w_hat), w_hat_ref, torch.float32, "reconstruction of the codes")
    dw64 = host(dw)
    assert_close(host(coef), oqw.coefficients(dw64), torch.float32, "coefficients")
    e = err.cpu().numpy()
    assert np.allclose(e, oqw.channel_error(dw64), rtol=1e-12, atol=0.0)
    counts = hit.qwha_allocate(e, d["budget"], d["k_min"], n)
    assert np.array_equal(counts, oqw.allocate(e, d["budget"], d["k_min"], n))
    assert int(counts.sum()) == d["budget"] and counts.min() >= d["k_min"]
    off = np.zeros(rows + 1, np.int64)
    off[1:] = np.cumsum(counts)
    cols, vals = hit.qwha_select(coef, torch.from_numpy(off).cuda())
    torch.cuda.synchronize()
    f = coef.cpu().numpy().astype(np.float64)
    woff, wcols = oqw.select(f, counts)
    assert np.array_equal(cols.cpu().numpy(), wcols)
    assert np.array_equal(vals.cpu().numpy().astype(np.float64), oqw.direct_values(f, woff, wcols))
    # the selected coefficients expand back through the one-sided adapter to
    # the best k-term approximation of dW: reconstruction error = dropped energy
    vfix, cfix = oqw.to_fixed_width(woff, wcols, oqw.direct_values(f, woff, wcols))
    approx = hit.wht_expand(to_gpu_f32(vfix[None]), torch.from_numpy(cfix[None]).cuda(), n, 1 / np.sqrt(n))[0]
    torch.cuda.synchronize()
    kept = np.zeros_like(f)
    row_of = np.repeat(np.arange(rows), counts)
    kept[row_of, wcols] = f[row_of, wcols]
    assert_close(host(approx), oh.irht_rows(kept, None), torch.float32, "adapter from the selection")
