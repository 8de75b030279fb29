"""GPU parity of the fused d = 5120 randomized transform + 4-bit group
quantization (rht_mixed_quantize_pack, through the C ABI) against the oracle:
oracle.butterfly.rht_mixed with the schedule (8, 8, 8, 5, 2) (Hadamard blocks
for the power-of-two radices, the seeded QR mixer for radix 5) followed by the
scalar fp32 quantizer.  Codes bit-exact outside the rounding-boundary window
(excused ones capped at 1e-5), scales within 1e-6."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import butterfly as ob
from oracle import quant as oq
from tests._parity import check_quant, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu


def oracle_codes(d, x, signs):
    blocks = ob.rht_stage_blocks(d["radices"], d["mixers"])
    return oq.quantize(ob.rht_mixed(x, signs, d["radices"], blocks), 4, 128)


def test_mixed_workload_full_size():
    """fp32 4096 x 5120, N(0, 0.02) with 0.1 % outliers x50, Rademacher signs:
    every row against the oracle, in the launch configuration the benchmark times."""
    d = synth.mixed_rht_int4()
    codes, scales = hit.rht_mixed_quantize_pack(to_gpu_f32(d["x"]), to_gpu_i8(d["signs"]), d["mixers"][5][0])
    torch.cuda.synchronize()
    check_quant(codes, scales, oracle_codes(d, d["x"], d["signs"]), 4, 5120)


@pytest.mark.parametrize("rows", [1, 7, 149, 300])
def test_ragged_rows_no_signs_and_padded_pitch(rows):
    d = synth.mixed_rht_int4(rows=rows, seed=50 + rows)
    # padded rows (leading dimension 5120 + 64), no signs
    wide = np.zeros((rows, 5184), np.float32)
    wide[:, :5120] = d["x"]
    xg = to_gpu_f32(wide)[:, :5120]
    codes, scales = hit.rht_mixed_quantize_pack(xg, None, d["mixers"][5][0])
    torch.cuda.synchronize()
    check_quant(codes, scales, oracle_codes(d, d["x"], np.ones(5120, np.int8)), 4, 5120)


def test_zero_rows_and_identity_mixer():
    """An all-zero row gives zero scales and offset codes; with G_5 = I the
    transform is H_512 (x) I_5 (x) H_2 / 32 applied to the signed input."""
    d = synth.mixed_rht_int4(rows=20, seed=77)
    x = d["x"].copy()
    x[4] = 0.0
    eye = np.eye(5, dtype=np.float32)
    dd = dict(d)
    dd["mixers"] = {5: eye[None]}
    codes, scales = hit.rht_mixed_quantize_pack(to_gpu_f32(x), to_gpu_i8(d["signs"]), eye)
    torch.cuda.synchronize()
    check_quant(codes, scales, oracle_codes(dd, x, d["signs"]), 4, 5120)
    assert float(scales[4].abs().max()) == 0.0
    assert bool((codes[4] == 0x88).all())
