"""GPU parity of butterfly_apply_tc (window matrices composed on the device,
bf16 x bf16 -> fp32 tensor-core passes, bf16 between passes; through the C
ABI) against the float64 oracle, with the bf16 tolerance (max over rows of
max |error| / max |reference row| <= 2e-2)."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import butterfly as ob
from tests._parity import assert_close, host, to_gpu_bf16, to_gpu_f32

pytestmark = pytest.mark.gpu


def blocks_for(radices, shared=False, seed=0):
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    return [synth.seeded_orthogonal_blocks(rng, 1 if shared else d // b, b) for b in radices]


def bf16_input(shape, seed):
    x = np.random.default_rng(seed).standard_normal(shape).astype(np.float32)
    bits = synth.to_bf16_bits(x)
    return bits, synth.bf16_bits_to_f32(bits)


@pytest.mark.parametrize("radices", [(4, 16, 8), (16, 16), (2, 64), (7, 16, 16, 8), (8, 8, 4, 4)])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_rows(radices, transpose, out_dtype):
    d = int(np.prod(radices))
    blocks = blocks_for(radices, seed=d)
    bits, xf = bf16_input((300, d), d)               # 300 rows: a ragged last row tile
    y = hit.butterfly_apply_tc(to_gpu_bf16(bits), radices, [to_gpu_f32(b) for b in blocks], axis=1,
                               transpose=transpose, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = ob.apply_stages(xf, radices, blocks, transpose)
    assert_close(host(y), ref, torch.bfloat16, f"rows {radices} T={transpose}")


@pytest.mark.parametrize("radices", [(7, 16, 16, 8), (4, 16, 8), (2, 16, 8, 8), (8, 8, 16), (16, 8, 16), (16, 4, 8)])
@pytest.mark.parametrize("transpose", [False, True])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_rows_strided_windows(radices, transpose, out_dtype):
    """Runs whose digits sit at a stride along the rows (SIMT passes inside the
    tensor-core plan) next to contiguous tensor-core windows, 264 rows (a
    ragged last 128-row tile)."""
    d = int(np.prod(radices))
    blocks = blocks_for(radices, seed=d + 5)
    bits, xf = bf16_input((264, d), d + 5)
    y = hit.butterfly_apply_tc(to_gpu_bf16(bits), radices, [to_gpu_f32(b) for b in blocks], axis=1,
                               transpose=transpose, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = ob.apply_stages(xf, radices, blocks, transpose)
    assert_close(host(y), ref, torch.bfloat16, f"strided rows {radices} T={transpose}")


@pytest.mark.parametrize("rows,radices", [(40, (7, 16, 8, 8, 8, 2, 2)), (5, (7, 16, 16, 8)), (33, (4, 16, 8, 4, 8))])
@pytest.mark.parametrize("transpose", [False, True])
def test_rows_strided_shapes(rows, radices, transpose):
    """Strided two-digit runs with more (lo group, hi) keys than SMs (the
    (7, 16) run at stride 2048: 256 keys), fewer rows than one 32-row tile,
    and a run whose boxes reach past the last hi block; fp32 results."""
    d = int(np.prod(radices))
    blocks = blocks_for(radices, seed=d + 11)
    bits, xf = bf16_input((rows, d), d + 11)
    y = hit.butterfly_apply_tc(to_gpu_bf16(bits), radices, [to_gpu_f32(b) for b in blocks], axis=1,
                               transpose=transpose, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = ob.apply_stages(xf, radices, blocks, transpose)
    assert_close(host(y), ref, torch.bfloat16, f"strided rows {radices} x {rows} T={transpose}")


@pytest.mark.parametrize("radices", [(16, 16, 16), (8, 16), (2, 4, 16), (16, 8, 2), (4, 32, 2)])
@pytest.mark.parametrize("transpose", [False, True])
def test_columns(radices, transpose):
    m = int(np.prod(radices))
    blocks = blocks_for(radices, seed=m + 1)
    bits, xf = bf16_input((m, 200), m)               # 200 columns: a ragged last column tile
    y = hit.butterfly_apply_tc(to_gpu_bf16(bits), radices, [to_gpu_f32(b) for b in blocks], axis=0,
                               transpose=transpose)
    torch.cuda.synchronize()
    ref = ob.apply_stages_cols(xf, radices, blocks, transpose)
    assert_close(host(y), ref, torch.bfloat16, f"cols {radices} T={transpose}")


def test_shared_blocks_and_padded_pitch():
    radices = (4, 8, 16)
    blocks = blocks_for(radices, shared=True, seed=9)
    bits, xf = bf16_input((64, 512), 3)
    wide = torch.zeros((64, 512 + 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :512] = to_gpu_bf16(bits)
    out = torch.zeros((64, 512 + 32), dtype=torch.bfloat16, device="cuda")
    hit.butterfly_apply_tc(wide[:, :512], radices, [to_gpu_f32(b) for b in blocks], out=out[:, :512])
    torch.cuda.synchronize()
    assert_close(host(out[:, :512]), ob.apply_stages(xf, radices, blocks), torch.bfloat16, "shared, padded")
    assert float(out[:, 512:].abs().max()) == 0.0, "columns past n were written"


def test_two_sided_butterfly_workload_tensor_cores():
    """bf16 4096 x 14336: R_in (7,16,16,8) along rows, then R_out (16,16,16)
    along columns, bf16 between the two, in the launch configuration the
    benchmark times; 12 output rows against the float64 oracle."""
    d = synth.two_sided_butterfly()
    x = to_gpu_bf16(d["x_bf16"])
    bi = [to_gpu_f32(b) for b in d["blocks_in"]]
    bo = [to_gpu_f32(b) for b in d["blocks_out"]]
    mid = hit.butterfly_apply_tc(x, d["radices_in"], bi, axis=1)
    y = hit.butterfly_apply_tc(mid, d["radices_out"], bo, axis=0)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 17, 2048, 4095, 3000, 64, 65, 66, 1234, 999, 4000])
    r_out = ob.dense(d["radices_out"], d["blocks_out"])
    w = synth.bf16_bits_to_f32(d["x_bf16"]).astype(np.float64)
    ref = ob.apply_stages(r_out[rows] @ w, d["radices_in"], d["blocks_in"])
    assert_close(host(y[rows.tolist()]), ref, torch.bfloat16, "two-sided butterfly (tensor cores)")
