"""GPU parity of the fused RHT + group quantization + packing and of the
dequantize + inverse path, one- and two-sided (through the C ABI)."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import hadamard as oh
from oracle import quant as oq
from tests._parity import MSE_REL, assert_close, check_quant, host, to_gpu_bf16, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu


def weights(rows, n, seed):
    d = synth.weight_rht_int4(rows=rows, n=n, seed=seed)
    return d["x"], d["signs"]


@pytest.mark.parametrize("logn", [5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_one_sided_every_length(logn, bits):
    n = 1 << logn
    rows = max(3, (1 << 17) // n) + 1  # >= 128K elements, ragged against the CTA row count
    x, s = weights(rows, n, 10 * logn + bits)
    group = min(n, 128)
    codes, scales = hit.rht_quantize_pack(to_gpu_f32(x), to_gpu_i8(s), bits, group)
    torch.cuda.synchronize()
    if n > 8192:  # long rows: three rows through the column-blocked oracle
        ref = oq.quantize(oh.rht_rows_chunked(x[:3], s), bits, group)
        check_quant(codes[:3], scales[:3], ref, bits, n)
        yr = hit.dequant_inverse(codes, scales, n, bits, group, to_gpu_i8(s))
        torch.cuda.synchronize()
        u = oq.unpack(codes[:3].cpu().numpy(), bits, n)
        rec = oh.irht_rows_chunked(oq.dequantize(u, scales[:3].cpu().numpy(), bits, group), s)
        assert_close(host(yr[:3]), rec, torch.float32, "dequant+inverse (long rows)")
        return
    y64 = oh.rht_rows(x, s)
    ref = oq.quantize(y64, bits, group)
    check_quant(codes, scales, ref, bits, n)
    # dequant + inverse against the oracle's reconstruction from the oracle's codes
    yr = hit.dequant_inverse(codes, scales, n, bits, group, to_gpu_i8(s))
    torch.cuda.synchronize()
    u = oq.unpack(codes.cpu().numpy(), bits, n)
    rec = oh.irht_rows(oq.dequantize(u, scales.cpu().numpy(), bits, group), s)
    assert_close(host(yr), rec, torch.float32, "dequant+inverse")


@pytest.mark.parametrize("group", [32, 64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("logn", [8, 12, 13])
def test_group_sizes(group, logn):
    n = 1 << logn
    if group > n:
        pytest.skip("group larger than the row")
    x, s = weights(64, n, group + logn)
    for bits in (2, 3, 4):
        codes, scales = hit.rht_quantize_pack(to_gpu_f32(x), to_gpu_i8(s), bits, group)
        torch.cuda.synchronize()
        check_quant(codes, scales, oq.quantize(oh.rht_rows(x, s), bits, group), bits, n)
        yr = hit.dequant_inverse(codes, scales, n, bits, group, to_gpu_i8(s), out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        u = oq.unpack(codes.cpu().numpy(), bits, n)
        rec = oh.irht_rows(oq.dequantize(u, scales.cpu().numpy(), bits, group), s)
        assert_close(host(yr), rec, torch.bfloat16, "bf16 reconstruction")


def test_bf16_input_no_signs_and_zero_groups():
    n = 4096
    x, _ = weights(33, n, 7)
    x[3] = 0.0                      # all-zero row -> zero scales, codes = 2^(bits-1)
    x[5, :] = x[5, :] * 1e-30       # tiny values: subnormal-range scales take the exact path
    bits16 = synth.to_bf16_bits(x)
    xb = synth.bf16_bits_to_f32(bits16)
    for bits in (2, 3, 4):
        codes, scales = hit.rht_quantize_pack(to_gpu_bf16(bits16), None, bits, 128)
        torch.cuda.synchronize()
        check_quant(codes, scales, oq.quantize(oh.rht_rows(xb, None), bits, 128), bits, n)
        assert float(scales[3].abs().max()) == 0.0


def test_weight_workload_full_size():
    """fp32 4096 x 4096 weights with 0.1 % outliers x50, 4-bit, g = 128, at the
    full size in the launch configuration the benchmark times; 512 rows spread
    over the matrix are checked against the oracle."""
    d = synth.weight_rht_int4()
    x = to_gpu_f32(d["x"])
    codes, scales = hit.rht_quantize_pack(x, to_gpu_i8(d["signs"]), 4, 128)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(8), np.linspace(0, 4095, 504).astype(int)]))
    ref = oq.quantize(oh.rht_rows(d["x"][rows], d["signs"]), 4, 128)
    check_quant(codes[rows.tolist()], scales[rows.tolist()], ref, 4, 4096)


@pytest.mark.parametrize("rows,n", [(256, 1024), (2048, 512), (64, 8192)])
@pytest.mark.parametrize("bits", [2, 3])
def test_two_sided_small(rows, n, bits):
    d = synth.two_sided_lowbit(rows=rows, n=n, seed=rows + n + bits)
    xb = synth.bf16_bits_to_f32(d["x_bf16"])
    x = to_gpu_bf16(d["x_bf16"])
    rs, cs = to_gpu_i8(d["row_signs"]), to_gpu_i8(d["col_signs"])
    codes, scales = hit.rht_quantize_pack(x, rs, bits, 64, col_signs=cs)
    torch.cuda.synchronize()
    ref = oq.quantize(oh.two_sided(xb, d["row_signs"], d["col_signs"]), bits, 64)
    check_quant(codes, scales, ref, bits, n)
    y = hit.dequant_inverse(codes, scales, n, bits, 64, rs, col_signs=cs)
    yb = hit.dequant_inverse(codes, scales, n, bits, 64, rs, col_signs=cs, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    u = oq.unpack(codes.cpu().numpy(), bits, n)
    rec = oh.two_sided_inverse(oq.dequantize(u, scales.cpu().numpy(), bits, 64), d["row_signs"], d["col_signs"])
    assert_close(host(y), rec, torch.float32, "two-sided reconstruction")
    assert_close(host(yb), rec, torch.bfloat16, "two-sided bf16 reconstruction")


@pytest.mark.parametrize("bits", [2, 3])
def test_two_sided_lowbit_workload_full_size(bits):
    """bf16 8192 x 8192 with 0.05 % outliers x100, two-sided RHT, groups of 64,
    then dequant + inverse, at full size: every code and scale against the
    oracle's; 24 rows of the reconstruction against the oracle's inverse of the
    GPU's own codes; and the reconstruction MSE of the whole matrix against the
    MSE of the oracle's own round trip (its codes, its inverse) within 1e-4
    relative."""
    d = synth.two_sided_lowbit()
    x = to_gpu_bf16(d["x_bf16"])
    rs, cs = to_gpu_i8(d["row_signs"]), to_gpu_i8(d["col_signs"])
    codes, scales = hit.rht_quantize_pack(x, rs, bits, 64, col_signs=cs)
    y = hit.dequant_inverse(codes, scales, 8192, bits, 64, rs, col_signs=cs)
    torch.cuda.synchronize()
    xb = synth.bf16_bits_to_f32(d["x_bf16"]).astype(np.float64)
    ref = oq.quantize(oh.two_sided(xb, d["row_signs"], d["col_signs"]), bits, 64)
    check_quant(codes, scales, ref, bits, 8192)
    # Reconstruction of the GPU's own codes, sampled rows, by the oracle.
    rows = np.array([0, 1, 2, 1000, 4095, 4096, 7000, 8191] + list(range(100, 116)))
    u = oq.unpack(codes.cpu().numpy(), bits, 8192)
    yhat = oq.dequantize(u, scales.cpu().numpy(), bits, 64)
    rec_rows = oh.two_sided_inverse_rows_at(yhat, d["row_signs"], d["col_signs"], rows)
    assert_close(host(y[rows.tolist()]), rec_rows, torch.float32, "two-sided reconstruction rows")
    # Whole-matrix reconstruction MSE against the oracle's round trip.
    rec = oh.two_sided_inverse(oq.dequantize(ref["u"], ref["scales"], bits, 64), d["row_signs"], d["col_signs"])
    mse_oracle = float(((rec - xb) ** 2).mean())
    mse_gpu = float(((host(y) - xb) ** 2).mean())
    assert abs(mse_gpu - mse_oracle) <= MSE_REL * mse_oracle, f"MSE {mse_gpu:.9e} vs oracle {mse_oracle:.9e}"


@pytest.mark.parametrize("bits", [4, 2])
def test_activation_per_token_quant_full_size(bits):
    """Online activation path: bf16 8192 x 4096 tokens (0.5 * Student-t(3) with
    1 % of the columns x20), RHT along the hidden dimension with Rademacher
    signs, then one absmax scale per token (group = 4096), in the launch
    configuration the benchmark times; every code against the oracle."""
    d = synth.activation_rht()
    xb = synth.bf16_bits_to_f32(d["x_bf16"])
    codes, scales = hit.rht_quantize_pack(to_gpu_bf16(d["x_bf16"]), to_gpu_i8(d["signs"]), bits, 4096)
    torch.cuda.synchronize()
    assert scales.shape == (8192, 1)
    ref = oq.quantize(oh.rht_rows(xb, d["signs"]), bits, 4096)
    check_quant(codes, scales, ref, bits, 4096)
