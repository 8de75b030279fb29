"""Comparison helpers for the GPU parity tests (tolerances from the workload
statement: fp32 transforms within 1e-5 relative L2, bf16 within 2e-2 of each
row's max |value|, codes bit-exact outside a 1e-6 rounding-boundary window
with at most 1e-5 of the codes excused, scales within 1e-6 relative, and a
reconstruction MSE within 1e-4 relative of the oracle's own)."""
import numpy as np
import torch

from oracle import quant as oq
from synth import bf16_bits_to_f32

F32_REL_L2 = 1e-5
BF16_ROW_REL = 2e-2
SCALE_REL = 1e-6
EXCUSED_FRACTION = 1e-5
MSE_REL = 1e-4


def dev():
    return torch.device("cuda:0")


def to_gpu_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def to_gpu_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).to(dev()).view(torch.bfloat16)


def to_gpu_i8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int8)).to(dev())


def host(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> float64 numpy (bf16 widened exactly)."""
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def rel_l2(got, ref) -> float:
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(np.asarray(got, np.float64) - ref) / (den if den > 0 else 1.0))


def bf16_row_rel(got, ref) -> float:
    ref = np.asarray(ref, np.float64)
    d = np.abs(np.asarray(got, np.float64) - ref).max(axis=-1)
    m = np.abs(ref).max(axis=-1)
    return float((d / np.where(m > 0, m, 1.0)).max()) if ref.size else 0.0


def assert_close(got, ref, dtype: torch.dtype, what: str = ""):
    if dtype == torch.float32:
        e = rel_l2(got, ref)
        assert e <= F32_REL_L2, f"{what} rel-L2 {e:.3e} > {F32_REL_L2}"
    else:
        e = bf16_row_rel(got, ref)
        assert e <= BF16_ROW_REL, f"{what} bf16 row-max rel {e:.3e} > {BF16_ROW_REL}"
    return e


def check_quant(codes_gpu: torch.Tensor, scales_gpu: torch.Tensor, ref: dict, bits: int, n: int):
    """Codes bit-exact outside the boundary window, excused ones counted; scales
    within 1e-6 relative.  Returns (excused, total)."""
    u = oq.unpack(codes_gpu.cpu().numpy(), bits, n)
    mism = u != ref["u"]
    win = oq.boundary_window(ref["t"])
    outside = int((mism & ~win).sum())
    excused = int((mism & win).sum())
    total = u.size
    assert outside == 0, f"{outside} codes differ outside the rounding-boundary window"
    assert excused <= EXCUSED_FRACTION * total, f"{excused} excused codes > {EXCUSED_FRACTION} of {total}"
    s = scales_gpu.cpu().numpy().astype(np.float64)
    rs = ref["scales"].astype(np.float64)
    rel = np.abs(s - rs) / np.where(rs > 0, rs, 1.0)
    assert float(rel.max(initial=0.0)) <= SCALE_REL, f"scale rel err {rel.max():.3e}"
    assert np.all((rs == 0) == (s == 0))
    return excused, total
