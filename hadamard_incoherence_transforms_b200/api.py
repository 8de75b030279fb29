"""PyTorch-facing wrappers over the libhit C ABI.

Argument marshalling only: each function checks that tensors live on a CUDA
device, allocates outputs (and workspace) with torch, and passes raw device
pointers, leading dimensions and the current CUDA stream to the C entry point
of the same name.  All arithmetic runs in the library's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import HIT_BF16, HIT_F32, call, load

_DT = {torch.float32: HIT_F32, torch.bfloat16: HIT_BF16}


def _dt(t: torch.dtype) -> int:
    if t not in _DT:
        raise TypeError(f"unsupported dtype {t}; use float32 or bfloat16")
    return _DT[t]


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t


def _mat(t: torch.Tensor, name: str) -> torch.Tensor:
    _cuda(t, name)
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with unit stride along the last dimension")
    return t


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _signs(s: torch.Tensor | None, length: int, name: str) -> torch.Tensor | None:
    if s is None:
        return None
    _cuda(s, name)
    if s.dtype != torch.int8 or s.dim() != 1 or s.numel() != length or not s.is_contiguous():
        raise ValueError(f"{name} must be a contiguous int8 vector of length {length}")
    return s


def workspace_bytes(op: int, rows: int, n: int, dtype_out: torch.dtype, flags: int) -> int:
    return int(load().hit_workspace_bytes(op, rows, n, _dt(dtype_out), flags))


def _workspace(ws: torch.Tensor | None, need: int, device) -> torch.Tensor | None:
    if need == 0:
        return ws
    if ws is not None:
        return ws
    return torch.empty(need // 4 + 4, dtype=torch.float32, device=device)


def _rht(name: str, x, signs, axis, out, out_dtype, workspace):
    x = _mat(x, "x")
    rows, n = x.shape
    out_dtype = out_dtype or (out.dtype if out is not None else x.dtype)
    if out is None:
        out = torch.empty((rows, n), dtype=out_dtype, device=x.device)
    _mat(out, "out")
    if out.shape != x.shape or out.dtype != out_dtype:
        raise ValueError("out must match x's shape and out_dtype")
    s = _signs(signs, n if axis == 1 else rows, "signs")
    need = workspace_bytes(_lib.HIT_OP_RHT, rows, n, out_dtype, axis)
    ws = _workspace(workspace, need, x.device)
    call(name, x.data_ptr(), out.data_ptr(), rows, n, x.stride(0), out.stride(0), _dt(x.dtype), _dt(out_dtype),
         _ptr(s), axis, _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    return out


def rht_forward(x, signs=None, axis: int = 1, out=None, out_dtype=None, workspace=None):
    """y = H diag(signs) x / sqrt(len) along rows (axis=1) or columns (axis=0)."""
    return _rht("rht_forward", x, signs, axis, out, out_dtype, workspace)


def rht_inverse(x, signs=None, axis: int = 1, out=None, out_dtype=None, workspace=None):
    """x = diag(signs) H y / sqrt(len) along rows (axis=1) or columns (axis=0)."""
    return _rht("rht_inverse", x, signs, axis, out, out_dtype, workspace)


def butterfly_apply(x, radices, blocks, axis: int = 1, transpose: bool = False, out=None, out_dtype=None,
                    workspace=None):
    """y = R x (or R^T x) for the mixed-radix stride butterfly with per-stage blocks.

    blocks[t]: float32 CUDA tensor [G_t, b_t, b_t] with G_t = L / b_t or 1.
    """
    x = _mat(x, "x")
    rows, n = x.shape
    m = len(radices)
    if len(blocks) != m:
        raise ValueError("one block tensor per radix")
    out_dtype = out_dtype or (out.dtype if out is not None else x.dtype)
    if out is None:
        out = torch.empty((rows, n), dtype=out_dtype, device=x.device)
    _mat(out, "out")
    for t, b in enumerate(blocks):
        _cuda(b, f"blocks[{t}]")
        if b.dtype != torch.float32 or b.dim() != 3 or not b.is_contiguous():
            raise ValueError(f"blocks[{t}] must be contiguous float32 [G, b, b]")
    rad = (ctypes.c_int32 * m)(*[int(r) for r in radices])
    bptr = (ctypes.c_void_p * m)(*[b.data_ptr() for b in blocks])
    ng = (ctypes.c_int64 * m)(*[int(b.shape[0]) for b in blocks])
    need = workspace_bytes(_lib.HIT_OP_BUTTERFLY, rows, n, out_dtype, m)
    ws = _workspace(workspace, need, x.device)
    call("butterfly_apply", x.data_ptr(), out.data_ptr(), rows, n, x.stride(0), out.stride(0), _dt(x.dtype),
         _dt(out_dtype), m, ctypes.cast(rad, ctypes.c_void_p), ctypes.cast(bptr, ctypes.c_void_p),
         ctypes.cast(ng, ctypes.c_void_p), int(bool(transpose)), axis, _ptr(ws),
         0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    return out


def codes_shape(rows: int, n: int, bits: int) -> tuple[int, int]:
    return rows, n * bits // 8


def rht_quantize_pack(x, row_signs, bits: int, group: int, col_signs=None, codes=None, scales=None,
                      workspace=None):
    """Fused (one- or two-sided) RHT + group absmax RTN + packing.  Returns (codes, scales)."""
    x = _mat(x, "x")
    rows, n = x.shape
    if codes is None:
        codes = torch.empty(codes_shape(rows, n, bits), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, n // group), dtype=torch.float32, device=x.device)
    _cuda(codes, "codes")
    _cuda(scales, "scales")
    if not codes.is_contiguous() or codes.dtype != torch.uint8 or codes.shape != codes_shape(rows, n, bits):
        raise ValueError("codes must be contiguous uint8 [rows, n*bits/8]")
    if not scales.is_contiguous() or scales.dtype != torch.float32 or scales.shape != (rows, n // group):
        raise ValueError("scales must be contiguous float32 [rows, n/group]")
    rs = _signs(row_signs, n, "row_signs")
    cs = _signs(col_signs, rows, "col_signs")
    need = workspace_bytes(_lib.HIT_OP_QUANT, rows, n, torch.float32, 1 if cs is not None else 0)
    ws = _workspace(workspace, need, x.device)
    call("rht_quantize_pack", x.data_ptr(), rows, n, x.stride(0), _dt(x.dtype), _ptr(rs), _ptr(cs), bits, group,
         codes.data_ptr(), scales.data_ptr(), _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
         _stream(x.device))
    return codes, scales


def dequant_inverse(codes, scales, n: int, bits: int, group: int, row_signs, col_signs=None,
                    out_dtype=torch.float32, out=None, workspace=None):
    """Dequantize packed codes and apply the inverse (one- or two-sided) RHT."""
    _cuda(codes, "codes")
    _cuda(scales, "scales")
    rows = codes.shape[0]
    if codes.dtype != torch.uint8 or not codes.is_contiguous() or codes.shape != codes_shape(rows, n, bits):
        raise ValueError("codes must be contiguous uint8 [rows, n*bits/8]")
    if scales.dtype != torch.float32 or not scales.is_contiguous() or scales.shape != (rows, n // group):
        raise ValueError("scales must be contiguous float32 [rows, n/group]")
    if out is None:
        out = torch.empty((rows, n), dtype=out_dtype, device=codes.device)
    _mat(out, "out")
    rs = _signs(row_signs, n, "row_signs")
    cs = _signs(col_signs, rows, "col_signs")
    need = workspace_bytes(_lib.HIT_OP_DEQUANT, rows, n, out.dtype, 1 if cs is not None else 0)
    ws = _workspace(workspace, need, codes.device)
    call("dequant_inverse", codes.data_ptr(), scales.data_ptr(), rows, n, bits, group, _ptr(rs), _ptr(cs),
         out.data_ptr(), out.stride(0), _dt(out.dtype), _ptr(ws),
         0 if ws is None else ws.numel() * ws.element_size(), _stream(codes.device))
    return out


def _sparse_check(values, cols):
    _cuda(values, "values")
    _cuda(cols, "cols")
    if values.dim() != 3 or values.shape != cols.shape:
        raise ValueError("values and cols must both be [batch, rows, nnz]")
    if values.dtype != torch.float32 or cols.dtype != torch.int32:
        raise ValueError("values must be float32 and cols int32")
    if not values.is_contiguous() or not cols.is_contiguous():
        raise ValueError("values and cols must be contiguous")


def wht_expand(values, cols, n: int, scale: float, out=None):
    """dense[b, r, :] = scatter(values, cols)[b, r, :] @ H_n * scale (duplicates add)."""
    _sparse_check(values, cols)
    bsz, rows, nnz = values.shape
    if out is None:
        out = torch.empty((bsz, rows, n), dtype=torch.float32, device=values.device)
    _cuda(out, "out")
    if out.shape != (bsz, rows, n) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous float32 [batch, rows, n]")
    call("wht_expand_sparse", values.data_ptr(), cols.data_ptr(), bsz, rows, n, nnz, float(scale), out.data_ptr(),
         0, _stream(values.device))
    return out


def wht_gather(dense, cols, scale: float, out=None):
    """values[b, r, k] = (dense[b, r, :] @ H_n * scale)[cols[b, r, k]] (the adapter gradient)."""
    _cuda(dense, "dense")
    bsz, rows, n = dense.shape
    if out is None:
        out = torch.empty(cols.shape, dtype=torch.float32, device=dense.device)
    _sparse_check(out, cols)
    if dense.dtype != torch.float32 or not dense.is_contiguous():
        raise ValueError("dense must be contiguous float32 [batch, rows, n]")
    call("wht_expand_sparse", out.data_ptr(), cols.data_ptr(), bsz, rows, n, cols.shape[2], float(scale),
         dense.data_ptr(), 1, _stream(dense.device))
    return out


def wait_timeouts(reset: bool = True) -> int:
    """Bounded device waits that gave up on the current device since the last
    reset (synchronizes the device).  0 means every output written since then
    is defined."""
    n = ctypes.c_ulonglong(0)
    status = load().hit_wait_timeouts(ctypes.byref(n), int(bool(reset)))
    if status not in (_lib.HIT_OK, _lib.HIT_ETIMEOUT):
        raise _lib.HitError("hit_wait_timeouts", status, load().hit_last_error().decode(errors="replace"))
    return int(n.value)


def wait_selftest(limit_ns: int = 1_000_000, device=None) -> None:
    """Launch one warp whose bounded wait runs out after limit_ns (nothing
    completes its barrier); wait_timeouts() then counts it."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    call("hit_wait_selftest", int(limit_ns), _stream(dev))


def harp_n_params(b: int) -> int:
    """Learnable parameters per b x b HARP block: 0 (b = 1), 1 (b = 2), b(b-1)/2."""
    return 0 if b == 1 else 1 if b == 2 else b * (b - 1) // 2


def harp_blocks(theta, b: int, mixer=None, signs=None, theta_scale: float | None = None, groups: int | None = None,
                out=None):
    """Blocks [groups, b, b] of one HARP stage, B_c = Q(theta_c) G_b.

    theta: float32 [groups, P] or int8 [groups, P] (then theta_scale is the
    per-stage scale of the stored parameters); None for b = 1 (give groups).
    mixer: float32 [b, b] (None = Sylvester / sqrt(b) for powers of two).
    signs: int8 [b * groups] to fold the RHT sign vector into a first stage."""
    if theta is not None:
        _cuda(theta, "theta")
        if theta.dim() != 2 or theta.shape[1] != harp_n_params(b) or not theta.is_contiguous():
            raise ValueError(f"theta must be contiguous [groups, {harp_n_params(b)}]")
        groups = theta.shape[0]
        if theta.dtype == torch.int8:
            if theta_scale is None:
                raise ValueError("int8 theta needs theta_scale")
        elif theta.dtype != torch.float32:
            raise ValueError("theta must be float32 or int8")
    elif groups is None:
        raise ValueError("give theta or groups")
    dev = theta.device if theta is not None else torch.device("cuda", torch.cuda.current_device())
    if mixer is not None:
        _cuda(mixer, "mixer")
        if mixer.shape != (b, b) or mixer.dtype != torch.float32 or not mixer.is_contiguous():
            raise ValueError(f"mixer must be contiguous float32 [{b}, {b}]")
    if signs is not None:
        _cuda(signs, "signs")
        if signs.dtype != torch.int8 or signs.numel() != b * groups or not signs.is_contiguous():
            raise ValueError(f"signs must be contiguous int8 of length {b * groups}")
    if out is None:
        out = torch.empty((groups, b, b), dtype=torch.float32, device=dev)
    q = theta is not None and theta.dtype == torch.int8
    call("harp_blocks", None if q or theta is None else theta.data_ptr(), theta.data_ptr() if q else None,
         float(theta_scale or 1.0), groups, b, _ptr(mixer), _ptr(signs), out.data_ptr(), _stream(dev))
    return out


def rht_mixed_quantize_pack(x, signs, mixer5, bits: int = 4, group: int = 128, codes=None, scales=None):
    """d = 5120 rows: y = R diag(s) x with the schedule (8, 8, 8, 5, 2) (Hadamard
    blocks for the power-of-two radices, the given 5 x 5 orthogonal mixer for
    radix 5), then 4-bit absmax RTN in groups of 128.  Returns (codes, scales)."""
    x = _mat(x, "x")
    rows, n = x.shape
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    g = [float(v) for v in (mixer5.flatten().tolist() if hasattr(mixer5, "flatten") else mixer5)]
    if len(g) != 25:
        raise ValueError("mixer5 must have 25 entries (5 x 5, row-major)")
    gh = (ctypes.c_float * 25)(*g)
    if codes is None:
        codes = torch.empty(codes_shape(rows, n, bits), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((rows, n // group), dtype=torch.float32, device=x.device)
    s = _signs(signs, n, "signs")
    call("rht_mixed_quantize_pack", x.data_ptr(), rows, n, x.stride(0), _ptr(s), ctypes.cast(gh, ctypes.c_void_p),
         bits, group, codes.data_ptr(), scales.data_ptr(), _stream(x.device))
    return codes, scales


def wht_expand_2d(values, cols, n: int, scale: float, out=None):
    """dense[b] = (H_m / sqrt m) scatter(values, cols)[b] H_n * scale, m = values.shape[1]."""
    _sparse_check(values, cols)
    bsz, m, nnz = values.shape
    if out is None:
        out = torch.empty((bsz, m, n), dtype=torch.float32, device=values.device)
    _cuda(out, "out")
    if out.shape != (bsz, m, n) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be contiguous float32 [batch, m, n]")
    call("wht_expand_sparse_2d", values.data_ptr(), cols.data_ptr(), bsz, m, n, nnz, float(scale), out.data_ptr(), 0,
         None, 0, _stream(values.device))
    return out


def wht_gather_2d(dense, cols, scale: float, out=None, workspace=None):
    """values[b, r, k] = ((H_m / sqrt m) dense[b] H_n * scale)[r, cols[b, r, k]] (the gradient of wht_expand_2d)."""
    _cuda(dense, "dense")
    bsz, m, n = dense.shape
    if dense.dtype != torch.float32 or not dense.is_contiguous():
        raise ValueError("dense must be contiguous float32 [batch, m, n]")
    if out is None:
        out = torch.empty(cols.shape, dtype=torch.float32, device=dense.device)
    _sparse_check(out, cols)
    ws = workspace if workspace is not None else torch.empty(bsz * m * n, dtype=torch.float32, device=dense.device)
    call("wht_expand_sparse_2d", out.data_ptr(), cols.data_ptr(), bsz, m, n, cols.shape[2], float(scale),
         dense.data_ptr(), 1, ws.data_ptr(), ws.numel() * ws.element_size(), _stream(dense.device))
    return out


def row_norms(x, out=None):
    """||x_r||_2 per row of an fp32 matrix, accumulated in fp64 (float64 [rows])."""
    x = _mat(x, "x")
    rows, n = x.shape
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    if out is None:
        out = torch.empty(rows, dtype=torch.float64, device=x.device)
    call("row_norms", x.data_ptr(), rows, n, x.stride(0), out.data_ptr(), _stream(x.device))
    return out


def qwha_allocate(err, budget: int, k_min: int, n: int):
    """AdaAlloc budget split (host arithmetic): int64 numpy counts per row."""
    import numpy as np

    e = np.ascontiguousarray(np.asarray(err, dtype=np.float64))
    counts = np.zeros(e.shape[0], dtype=np.int64)
    call("qwha_allocate", e.ctypes.data_as(ctypes.c_void_p), e.shape[0], int(budget), int(k_min), int(n),
         counts.ctypes.data_as(ctypes.c_void_p))
    return counts


def qwha_select(f, offsets, cols=None, values=None):
    """Per-row top-|f| selection on the device (CSR offsets int64 [rows + 1] on the
    device); returns (cols int32, values float32) in ascending column order per row."""
    f = _mat(f, "f")
    rows, n = f.shape
    _cuda(offsets, "offsets")
    if offsets.dtype != torch.int64 or offsets.numel() != rows + 1 or not offsets.is_contiguous():
        raise ValueError("offsets must be contiguous int64 [rows + 1]")
    total = int(offsets[-1].item())
    if cols is None:
        cols = torch.empty(total, dtype=torch.int32, device=f.device)
    if values is None:
        values = torch.empty(total, dtype=torch.float32, device=f.device)
    call("qwha_select", f.data_ptr(), rows, n, f.stride(0), offsets.data_ptr(), cols.data_ptr(), values.data_ptr(),
         _stream(f.device))
    return cols, values


def butterfly_tc_workspace_bytes(rows: int, n: int, radices, axis: int = 1, transpose: bool = False) -> int:
    m = len(radices)
    rad = (ctypes.c_int32 * m)(*[int(r) for r in radices])
    return int(load().butterfly_tc_workspace_bytes(rows, n, axis, m, ctypes.cast(rad, ctypes.c_void_p),
                                                   int(bool(transpose))))


def butterfly_apply_tc(x, radices, blocks, axis: int = 1, transpose: bool = False, out=None, out_dtype=None,
                       workspace=None):
    """butterfly_apply on the tensor cores: bf16 input, window matrices composed on
    the device, bf16 x bf16 -> fp32 products per pass, bf16 between passes."""
    x = _mat(x, "x")
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bfloat16")
    rows, n = x.shape
    m = len(radices)
    if len(blocks) != m:
        raise ValueError("one block tensor per radix")
    out_dtype = out_dtype or (out.dtype if out is not None else x.dtype)
    if out is None:
        out = torch.empty((rows, n), dtype=out_dtype, device=x.device)
    _mat(out, "out")
    for t, b in enumerate(blocks):
        _cuda(b, f"blocks[{t}]")
        if b.dtype != torch.float32 or b.dim() != 3 or not b.is_contiguous():
            raise ValueError(f"blocks[{t}] must be contiguous float32 [G, b, b]")
    rad = (ctypes.c_int32 * m)(*[int(r) for r in radices])
    bptr = (ctypes.c_void_p * m)(*[b.data_ptr() for b in blocks])
    ng = (ctypes.c_int64 * m)(*[int(b.shape[0]) for b in blocks])
    need = butterfly_tc_workspace_bytes(rows, n, radices, axis, transpose)
    ws = workspace
    if ws is None and need > 0:
        ws = torch.empty(need // 4 + 64, dtype=torch.float32, device=x.device)
    call("butterfly_apply_tc", x.data_ptr(), out.data_ptr(), rows, n, x.stride(0), out.stride(0), _dt(x.dtype),
         _dt(out_dtype), m, ctypes.cast(rad, ctypes.c_void_p), ctypes.cast(bptr, ctypes.c_void_p),
         ctypes.cast(ng, ctypes.c_void_p), int(bool(transpose)), axis, _ptr(ws),
         0 if ws is None else ws.numel() * ws.element_size(), _stream(x.device))
    return out
