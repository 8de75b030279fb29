"""rht_quantize_pack_noalloc against rht_quantize_pack (GPU, through the C ABI).

The no-allocation entry point exists for callers that cannot call cudaMalloc
-- for example plug-ins whose host application owns all device memory, or
latency-critical paths that must not block on the allocator -- and therefore
cannot hand the two-sided quantizer a workspace.  It keeps the intermediate
in the library's own static scratch array instead.  Its codes and scales must
equal those of the regular entry point (which gets a workspace from the
caller), on consecutive calls that reuse the array.

This module is named so that pytest collects it after every other test file.
"""
import ctypes

import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from hadamard_incoherence_transforms_b200 import _lib
from tests._parity import SCALE_REL, to_gpu_bf16, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu

MAX_ELEMS = 4194304  # HIT_NOALLOC_MAX_ELEMS in include/hit.h


def noalloc(x, rs, cs, bits, group, codes, scales):
    lib = _lib.load()
    rows, n = x.shape
    stream = torch.cuda.current_stream().cuda_stream
    dt = _lib.HIT_BF16 if x.dtype == torch.bfloat16 else _lib.HIT_F32
    return lib.rht_quantize_pack_noalloc(
        ctypes.c_void_p(x.data_ptr()), rows, n, x.stride(0), dt,
        ctypes.c_void_p(rs.data_ptr()), None if cs is None else ctypes.c_void_p(cs.data_ptr()), bits, group,
        ctypes.c_void_p(codes.data_ptr()), ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(stream))


@pytest.mark.parametrize("bits", [3, 4])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(bits):
    for call, (rows, n) in enumerate([(1024, 2048), (2048, 2048)]):  # the second call reuses the array
        d = synth.two_sided_lowbit(rows=rows, n=n, seed=100 * bits + call)
        x = to_gpu_bf16(d["x_bf16"])
        rs, cs = to_gpu_i8(d["row_signs"]), to_gpu_i8(d["col_signs"])
        ref_codes, ref_scales = hit.rht_quantize_pack(x, rs, bits, 64, col_signs=cs)
        codes = torch.full_like(ref_codes, 0xAA)
        scales = torch.full_like(ref_scales, -1.0)
        assert noalloc(x, rs, cs, bits, 64, codes, scales) == _lib.HIT_OK
        torch.cuda.synchronize()
        assert torch.equal(codes, ref_codes), f"call {call}: codes differ"
        rel = (scales.double() - ref_scales.double()).abs() / ref_scales.double().clamp_min(1e-30)
        assert float(rel.max()) <= SCALE_REL, f"call {call}: scales differ"


def test_noalloc_one_sided_and_size_limit():
    d = synth.two_sided_lowbit(rows=256, n=4096, seed=7)
    x = to_gpu_bf16(d["x_bf16"])
    rs = to_gpu_i8(d["row_signs"])
    ref_codes, ref_scales = hit.rht_quantize_pack(x, rs, 4, 128)
    codes, scales = torch.empty_like(ref_codes), torch.empty_like(ref_scales)
    assert noalloc(x, rs, None, 4, 128, codes, scales) == _lib.HIT_OK
    torch.cuda.synchronize()
    assert torch.equal(codes, ref_codes) and torch.equal(scales, ref_scales)
    # two-sided problems larger than the static array are refused before any launch
    big = torch.empty((4096, 2048), dtype=torch.bfloat16, device="cuda")
    assert big.numel() > MAX_ELEMS
    cs = to_gpu_i8(np.ones(4096, np.int8))
    bc = torch.empty((4096, 1024), dtype=torch.uint8, device="cuda")
    bs = torch.empty((4096, 32), dtype=torch.float32, device="cuda")
    rs2 = to_gpu_i8(np.ones(2048, np.int8))
    assert noalloc(big, rs2, cs, 4, 64, bc, bs) == _lib.HIT_EWORKSPACE
    assert b"static scratch" in _lib.load().hit_last_error()


def test_noalloc_full_array_fp32_and_padded_rows():
    """An fp32 source (the column pass's 8-column fp32 strips) of exactly
    HIT_NOALLOC_MAX_ELEMS elements, which writes the last bytes of the static
    array, then a bf16 source whose rows are padded (leading dimension > n)."""
    d = synth.weight_rht_int4(rows=4096, n=1024, seed=31)
    x = to_gpu_f32(d["x"])
    assert x.numel() == MAX_ELEMS
    rs = to_gpu_i8(d["signs"])
    cs = to_gpu_i8(np.where(np.random.default_rng(32).random(4096) < 0.5, -1, 1).astype(np.int8))
    for _ in range(2):
        ref_codes, ref_scales = hit.rht_quantize_pack(x, rs, 4, 128, col_signs=cs)
        codes = torch.full_like(ref_codes, 0x5A)
        scales = torch.full_like(ref_scales, -1.0)
        assert noalloc(x, rs, cs, 4, 128, codes, scales) == _lib.HIT_OK
        torch.cuda.synchronize()
        assert torch.equal(codes, ref_codes)
        rel = (scales.double() - ref_scales.double()).abs() / ref_scales.double().clamp_min(1e-30)
        assert float(rel.max()) <= SCALE_REL
    e = synth.two_sided_lowbit(rows=1024, n=2048, seed=33)
    wide = torch.zeros((1024, 2048 + 64), dtype=torch.bfloat16, device="cuda")
    wide[:, :2048] = to_gpu_bf16(e["x_bf16"])
    xp = wide[:, :2048]
    assert xp.stride(0) == 2048 + 64
    rs2, cs2 = to_gpu_i8(e["row_signs"]), to_gpu_i8(e["col_signs"])
    ref_codes, ref_scales = hit.rht_quantize_pack(xp, rs2, 3, 64, col_signs=cs2)
    codes, scales = torch.empty_like(ref_codes), torch.empty_like(ref_scales)
    assert noalloc(xp, rs2, cs2, 3, 64, codes, scales) == _lib.HIT_OK
    torch.cuda.synchronize()
    assert torch.equal(codes, ref_codes)
    rel = (scales.double() - ref_scales.double()).abs() / ref_scales.double().clamp_min(1e-30)
    assert float(rel.max()) <= SCALE_REL
