"""GPU parity of butterfly_apply (mixed-radix stride stages) against the oracle."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import butterfly as ob
from oracle import hadamard as oh
from tests._parity import assert_close, host, to_gpu_bf16, to_gpu_f32
from tests.test_oracle_hadamard import popcount_hadamard

pytestmark = pytest.mark.gpu


def blocks_for(radices, shared=False, seed=0):
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    return [synth.seeded_orthogonal_blocks(rng, 1 if shared else d // b, b) for b in radices]


@pytest.mark.parametrize("radices", [(3, 4), (7, 16, 8), (2, 3, 5), (16, 16), (64,), (5, 1, 6), (8, 8, 8, 5, 2)])
@pytest.mark.parametrize("axis", [1, 0])
@pytest.mark.parametrize("transpose", [False, True])
def test_small_schedules(radices, axis, transpose):
    d = int(np.prod(radices))
    blocks = blocks_for(radices, seed=d)
    other = 37
    shape = (other, d) if axis == 1 else (d, other)
    x = np.random.default_rng(d + axis).standard_normal(shape).astype(np.float32)
    y = hit.butterfly_apply(to_gpu_f32(x), radices, [to_gpu_f32(b) for b in blocks], axis=axis, transpose=transpose)
    torch.cuda.synchronize()
    if axis == 1:
        ref = ob.apply_stages(x, radices, blocks, transpose)
    else:
        ref = ob.apply_stages_cols(x, radices, blocks, transpose)
    assert_close(host(y), ref, torch.float32, f"{radices} axis {axis}")


def test_shared_blocks_and_bf16():
    radices = (4, 8, 2)
    blocks = blocks_for(radices, shared=True, seed=3)
    x = np.random.default_rng(1).standard_normal((20, 64)).astype(np.float32)
    bits = synth.to_bf16_bits(x)
    y = hit.butterfly_apply(to_gpu_bf16(bits), radices, [to_gpu_f32(b) for b in blocks])
    torch.cuda.synchronize()
    ref = ob.apply_stages(synth.bf16_bits_to_f32(bits), radices, blocks)
    assert_close(host(y), ref, torch.bfloat16, "shared bf16")


def test_hadamard_blocks_recover_the_rht():
    radices = (16, 16, 16)
    h16 = (popcount_hadamard(16) / 4.0).astype(np.float32)     # input blocks, not from the oracle
    blocks = [np.broadcast_to(h16, (256, 16, 16)).copy() for _ in radices]
    x = np.random.default_rng(2).standard_normal((9, 4096)).astype(np.float32)
    y = hit.butterfly_apply(to_gpu_f32(x), radices, [to_gpu_f32(b) for b in blocks])
    z = hit.rht_forward(to_gpu_f32(x))
    torch.cuda.synchronize()
    assert_close(host(y), oh.rht_rows(x, None), torch.float32, "hadamard blocks")
    assert_close(host(y), host(z), torch.float32, "butterfly vs rht")


def test_two_sided_butterfly_workload_full_size():
    """bf16 4096 x 14336: R_in (7,16,16,8) along rows, then R_out (16,16,16)
    along columns, fp32 between the two; 12 output rows against the oracle."""
    d = synth.two_sided_butterfly()
    x = to_gpu_bf16(d["x_bf16"])
    bi = [to_gpu_f32(b) for b in d["blocks_in"]]
    bo = [to_gpu_f32(b) for b in d["blocks_out"]]
    mid = hit.butterfly_apply(x, d["radices_in"], bi, axis=1, out_dtype=torch.float32)
    y = hit.butterfly_apply(mid, d["radices_out"], bo, axis=0, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 17, 2048, 4095, 3000, 64, 65, 66, 1234, 999, 4000])
    r_out = ob.dense(d["radices_out"], d["blocks_out"])          # 4096 x 4096
    w = synth.bf16_bits_to_f32(d["x_bf16"]).astype(np.float64)
    comb = r_out[rows] @ w                                        # rows of R_out W
    ref = ob.apply_stages(comb, d["radices_in"], d["blocks_in"])  # then R_in along rows
    assert_close(host(y[rows.tolist()]), ref, torch.bfloat16, "two-sided butterfly")
