"""The C ABI library loads, exports every symbol include/hit.h declares, and
rejects bad arguments on the host before any CUDA call (CPU only)."""
import ctypes
import os
import re

import pytest

from hadamard_incoherence_transforms_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hit.h")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"HIT_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from hadamard_incoherence_transforms_b200 import build

        build.build()
    return _lib.load()


def test_header_declares_the_six_operations():
    names = set(declared_symbols())
    for op in ("rht_forward", "rht_inverse", "butterfly_apply", "rht_quantize_pack", "dequant_inverse",
               "wht_expand_sparse"):
        assert op in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 10
    for name in names:
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_status_strings_and_version(lib):
    assert lib.hit_version() == 100
    assert lib.hit_status_string(0) == b"ok"
    assert b"workspace" in lib.hit_status_string(-5)


def test_workspace_sizes(lib):
    assert lib.hit_workspace_bytes(_lib.HIT_OP_QUANT, 8192, 8192, 0, 1) == 8192 * 8192 * 4
    assert lib.hit_workspace_bytes(_lib.HIT_OP_QUANT, 8192, 8192, 0, 0) == 0
    assert lib.hit_workspace_bytes(_lib.HIT_OP_DEQUANT, 256, 64, 0, 1) == 0
    assert lib.hit_workspace_bytes(_lib.HIT_OP_DEQUANT, 256, 64, 1, 1) == 256 * 64 * 4
    assert lib.hit_workspace_bytes(_lib.HIT_OP_RHT, 256, 64, 1, 0) == 256 * 64 * 4
    assert lib.hit_workspace_bytes(_lib.HIT_OP_RHT, 128, 64, 1, 0) == 0
    assert lib.hit_workspace_bytes(_lib.HIT_OP_BUTTERFLY, 16, 12, 1, 2) == 16 * 12 * 4


FAKE = 0x10000  # a 64 KiB-aligned address that is never dereferenced: checks fail first


def status(lib, name, *args):
    return getattr(lib, name)(*args)


def test_rht_rejects_bad_arguments_on_host(lib):
    # n not a power of two
    assert status(lib, "rht_forward", FAKE, FAKE, 4, 12, 12, 12, 0, 0, None, 1, None, 0, None) == _lib.HIT_EINVAL
    # NULL x
    assert status(lib, "rht_forward", None, FAKE, 4, 16, 16, 16, 0, 0, None, 1, None, 0, None) == _lib.HIT_EINVAL
    # misaligned base
    assert status(lib, "rht_forward", FAKE + 4, FAKE, 4, 16, 16, 16, 0, 0, None, 1, None, 0, None) == _lib.HIT_EALIGN
    # leading dimension not a multiple of 16 bytes
    assert status(lib, "rht_forward", FAKE, FAKE, 4, 16, 17, 16, 0, 0, None, 1, None, 0, None) == _lib.HIT_EALIGN
    # too long a row
    assert status(lib, "rht_forward", FAKE, FAKE, 1, 65536, 65536, 65536, 0, 0, None, 1, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    # bad dtype / axis
    assert status(lib, "rht_forward", FAKE, FAKE, 4, 16, 16, 16, 7, 0, None, 1, None, 0, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, "rht_inverse", FAKE, FAKE, 4, 16, 16, 16, 0, 0, None, 2, None, 0, None) == _lib.HIT_EINVAL
    # columns: bf16 output over 128 rows needs workspace
    assert status(lib, "rht_forward", FAKE, FAKE, 256, 16, 16, 16, 0, 1, None, 0, None, 0, None) == \
        _lib.HIT_EWORKSPACE
    assert b"workspace" in lib.hit_last_error()
    # empty input is a no-op that succeeds without touching the device
    assert status(lib, "rht_forward", FAKE, FAKE, 0, 16, 16, 16, 0, 0, None, 1, None, 0, None) == _lib.HIT_OK


def test_quant_rejects_bad_arguments_on_host(lib):
    q = "rht_quantize_pack"
    assert status(lib, q, FAKE, 4, 4096, 4096, 0, None, None, 5, 128, FAKE, FAKE, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, q, FAKE, 4, 4096, 4096, 0, None, None, 4, 100, FAKE, FAKE, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, q, FAKE, 4, 4096, 4096, 0, None, None, 4, 16, FAKE, FAKE, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, q, FAKE, 4, 16, 16, 0, None, None, 4, 32, FAKE, FAKE, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, q, FAKE, 4, 4096, 4096, 0, None, None, 4, 128, FAKE + 8, FAKE, None, 0, None) == \
        _lib.HIT_EALIGN
    assert status(lib, q, FAKE, 4, 4096, 4096, 0, None, None, 4, 128, None, FAKE, None, 0, None) == \
        _lib.HIT_EINVAL
    # two-sided needs power-of-two rows and a workspace
    assert status(lib, q, FAKE, 6, 4096, 4096, 0, None, FAKE, 4, 128, FAKE, FAKE, FAKE, 1 << 30, None) == \
        _lib.HIT_EINVAL
    assert status(lib, q, FAKE, 8, 4096, 4096, 0, None, FAKE, 4, 128, FAKE, FAKE, None, 0, None) == \
        _lib.HIT_EWORKSPACE
    d = "dequant_inverse"
    assert status(lib, d, FAKE, FAKE, 4, 4096, 4, 128, None, None, None, 4096, 0, None, 0, None) == _lib.HIT_EINVAL
    assert status(lib, d, FAKE, FAKE, 8, 4096, 4, 128, None, FAKE, FAKE, 4096, 1, None, 0, None) == \
        _lib.HIT_EWORKSPACE


def test_butterfly_and_sparse_reject_bad_arguments_on_host(lib):
    rad = (ctypes.c_int32 * 2)(3, 5)
    blk = (ctypes.c_void_p * 2)(FAKE, FAKE)
    ng = (ctypes.c_int64 * 2)(5, 3)
    args = [ctypes.cast(rad, ctypes.c_void_p), ctypes.cast(blk, ctypes.c_void_p), ctypes.cast(ng, ctypes.c_void_p)]
    assert status(lib, "butterfly_apply", FAKE, FAKE, 4, 16, 16, 16, 0, 0, 2, *args, 0, 1, None, 0, None) == \
        _lib.HIT_EINVAL  # 3*5 != 16
    bad_ng = (ctypes.c_int64 * 2)(4, 3)
    args2 = [args[0], args[1], ctypes.cast(bad_ng, ctypes.c_void_p)]
    assert status(lib, "butterfly_apply", FAKE, FAKE, 4, 15, 15, 15, 0, 0, 2, *args2, 0, 1, None, 0, None) == \
        _lib.HIT_EINVAL
    big = (ctypes.c_int32 * 1)(128)
    args3 = [ctypes.cast(big, ctypes.c_void_p), args[1], args[2]]
    assert status(lib, "butterfly_apply", FAKE, FAKE, 4, 128, 128, 128, 0, 0, 1, *args3, 0, 1, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    s = "wht_expand_sparse"
    assert status(lib, s, FAKE, FAKE, 1, 4, 4096, 0, ctypes.c_float(1.0), FAKE, 0, None) == _lib.HIT_EINVAL
    assert status(lib, s, FAKE, FAKE, 1, 4, 4000, 64, ctypes.c_float(1.0), FAKE, 0, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, s, FAKE, FAKE, 1, 4, 4096, 64, ctypes.c_float(1.0), FAKE, 2, None) == _lib.HIT_EINVAL
    assert status(lib, s, FAKE, FAKE, 1, 4, 4096, 64, ctypes.c_float(1.0), FAKE + 4, 0, None) == _lib.HIT_EALIGN
    assert status(lib, s, FAKE, FAKE, 0, 4, 4096, 64, ctypes.c_float(1.0), FAKE, 0, None) == _lib.HIT_OK


def test_binding_fails_loudly_without_cuda_tensors():
    import torch

    import hadamard_incoherence_transforms_b200 as hit

    with pytest.raises(ValueError):
        hit.rht_forward(torch.zeros(4, 16))


def test_wait_selftest_rejects_limits_on_the_host(lib):
    # outside [1 us, 1 s]: refused before any launch
    assert lib.hit_wait_selftest(0, None) == _lib.HIT_EINVAL
    assert lib.hit_wait_selftest(999, None) == _lib.HIT_EINVAL
    assert lib.hit_wait_selftest(1_000_000_001, None) == _lib.HIT_EINVAL
    assert b"timeout" in lib.hit_status_string(_lib.HIT_ETIMEOUT) or b"gave up" in lib.hit_status_string(-6)


def test_noalloc_checks_arguments_before_its_size_limit(lib):
    na = "rht_quantize_pack_noalloc"
    # a bad n, bits or group with a huge rows * n gets rht_quantize_pack's own status
    assert status(lib, na, FAKE, 1 << 20, 3000, 3000, 0, None, FAKE, 4, 128, FAKE, FAKE, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, na, FAKE, 1 << 20, 4096, 4096, 0, None, FAKE, 5, 128, FAKE, FAKE, None) == \
        _lib.HIT_EUNSUPPORTED
    assert status(lib, na, FAKE, 1 << 20, 4096, 4096, 0, None, FAKE, 4, 100, FAKE, FAKE, None) == \
        _lib.HIT_EUNSUPPORTED
    # odd (non power-of-two) rows for a two-sided call
    assert status(lib, na, FAKE, 3 << 20, 4096, 4096, 0, None, FAKE, 4, 128, FAKE, FAKE, None) == _lib.HIT_EINVAL
    # rows * n that would wrap around 64 bits is rejected, not wrapped
    assert status(lib, na, FAKE, 1 << 24, 32768, 32768, 0, None, FAKE, 4, 128, FAKE, FAKE, None) == \
        _lib.HIT_EWORKSPACE
    # valid arguments one row above the limit: refused, launching nothing
    assert status(lib, na, FAKE, 8192, 1024, 1024, 0, None, FAKE, 4, 128, FAKE, FAKE, None) == _lib.HIT_EWORKSPACE
    assert b"static scratch" in lib.hit_last_error()
    # no rows: nothing to do
    assert status(lib, na, FAKE, 0, 1024, 1024, 0, None, FAKE, 4, 128, FAKE, FAKE, None) == _lib.HIT_OK


def test_harp_blocks_rejects_bad_arguments_on_host(lib):
    h = "harp_blocks"
    one = ctypes.c_float(1.0)
    assert status(lib, h, FAKE, None, one, 4, 17, None, None, FAKE, None) == _lib.HIT_EUNSUPPORTED  # b > 16
    assert status(lib, h, FAKE, None, one, 4, 0, None, None, FAKE, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, h, FAKE, FAKE, one, 4, 4, None, None, FAKE, None) == _lib.HIT_EINVAL  # both thetas
    assert status(lib, h, None, None, one, 4, 4, None, None, FAKE, None) == _lib.HIT_EINVAL  # neither
    assert status(lib, h, FAKE, None, one, 4, 5, None, None, FAKE, None) == _lib.HIT_EINVAL  # radix 5 needs a mixer
    assert status(lib, h, FAKE, None, one, 4, 4, None, None, None, None) == _lib.HIT_EINVAL  # no output
    assert status(lib, h, FAKE, None, one, 4, 4, None, None, FAKE + 2, None) == _lib.HIT_EALIGN
    assert status(lib, h, FAKE, None, one, 0, 4, None, None, FAKE, None) == _lib.HIT_OK  # no groups: nothing to do


def test_mixed_rejects_bad_arguments_on_host(lib):
    m = "rht_mixed_quantize_pack"
    g = (ctypes.c_float * 25)(*([1.0] + [0.0] * 24))
    gp = ctypes.cast(g, ctypes.c_void_p)
    assert status(lib, m, FAKE, 4, 4096, 4096, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, m, FAKE, 4, 5120, 5120, None, gp, 3, 128, FAKE, FAKE, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, m, FAKE, 4, 5120, 5120, None, gp, 4, 64, FAKE, FAKE, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, m, FAKE, 4, 5120, 5120, None, None, 4, 128, FAKE, FAKE, None) == _lib.HIT_EINVAL
    assert status(lib, m, FAKE, 4, 5120, 5121, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_EALIGN
    assert status(lib, m, FAKE + 4, 4, 5120, 5120, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_EALIGN
    assert status(lib, m, FAKE, 4, 5120, 5000, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_EINVAL
    g[3] = float("nan")
    assert status(lib, m, FAKE, 4, 5120, 5120, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_EINVAL
    assert status(lib, m, FAKE, 0, 5120, 5120, None, gp, 4, 128, FAKE, FAKE, None) == _lib.HIT_OK


def test_qwha_entry_points_reject_bad_arguments_on_host(lib):
    assert status(lib, "qwha_select", FAKE, 4, 3000, 3000, FAKE, FAKE, FAKE, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, "qwha_select", FAKE, 4, 4096, 4095, FAKE, FAKE, FAKE, None) == _lib.HIT_EINVAL
    assert status(lib, "qwha_select", FAKE + 4, 4, 4096, 4096, FAKE, FAKE, FAKE, None) == _lib.HIT_EALIGN
    assert status(lib, "qwha_select", FAKE, 0, 4096, 4096, FAKE, FAKE, FAKE, None) == _lib.HIT_OK
    assert status(lib, "row_norms", FAKE, 4, 4098, 4098, FAKE, None) == _lib.HIT_EINVAL
    assert status(lib, "row_norms", FAKE + 4, 4, 4096, 4096, FAKE, None) == _lib.HIT_EALIGN
    w = "wht_expand_sparse_2d"
    one = ctypes.c_float(1.0)
    assert status(lib, w, FAKE, FAKE, 1, 300, 4096, 64, one, FAKE, 0, None, 0, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, w, FAKE, FAKE, 1, 256, 4000, 64, one, FAKE, 0, None, 0, None) == _lib.HIT_EUNSUPPORTED
    assert status(lib, w, FAKE, FAKE, 1, 256, 4096, 0, one, FAKE, 0, None, 0, None) == _lib.HIT_EINVAL
    assert status(lib, w, FAKE, FAKE, 1, 256, 4096, 64, one, FAKE, 2, None, 0, None) == _lib.HIT_EINVAL
    assert status(lib, w, FAKE, FAKE, 1, 256, 4096, 64, one, FAKE, 1, None, 0, None) == _lib.HIT_EWORKSPACE
    assert status(lib, w, FAKE, FAKE, 0, 256, 4096, 64, one, FAKE, 0, None, 0, None) == _lib.HIT_OK


def test_butterfly_tc_host_checks_and_workspace(lib):
    import ctypes as ct

    def ws(rows, n, axis, radices, transpose=0):
        r = (ct.c_int32 * len(radices))(*radices)
        return lib.butterfly_tc_workspace_bytes(rows, n, axis, len(radices), ct.cast(r, ct.c_void_p), transpose)

    # R_in of the butterfly workload: {2,3} on tensor cores (window 128), {0,1} a strided two-digit run
    # (no window matrix), one bf16 intermediate
    assert ws(4096, 14336, 1, (7, 16, 16, 8)) >= 14336 * 128 * 2 + 4096 * 14336 * 2
    # R_out: {0,1} (window 256 at stride 16) and {2} (block-diagonal windows of 128)
    assert ws(4096, 14336, 0, (16, 16, 16)) >= 4096 * 256 * 2 + 4096 * 128 * 2 + 4096 * 14336 * 2
    assert ws(4096, 14336, 0, (16, 16, 15)) == 0  # radices do not multiply to the length
    rad = (ct.c_int32 * 2)(16, 16)
    blk = (ct.c_void_p * 2)(FAKE, FAKE)
    ng = (ct.c_int64 * 2)(16, 16)
    args = [ct.cast(rad, ct.c_void_p), ct.cast(blk, ct.c_void_p), ct.cast(ng, ct.c_void_p)]
    t = "butterfly_apply_tc"
    # fp32 input is refused (tensor-core operands are bf16)
    assert status(lib, t, FAKE, FAKE + 0x100000, 8, 256, 256, 256, 0, 1, 2, *args, 0, 1, None, 0, None) == \
        _lib.HIT_EUNSUPPORTED
    # aliasing input and output
    assert status(lib, t, FAKE, FAKE, 8, 256, 256, 256, 1, 1, 2, *args, 0, 1, None, 0, None) == _lib.HIT_EINVAL
    # misaligned pitch
    assert status(lib, t, FAKE, FAKE + 0x100000, 8, 256, 260, 256, 1, 1, 2, *args, 0, 1, None, 0, None) == \
        _lib.HIT_EALIGN
    # no workspace for the window matrices
    assert status(lib, t, FAKE, FAKE + 0x100000, 8, 256, 256, 256, 1, 1, 2, *args, 0, 1, None, 0, None) == \
        _lib.HIT_EWORKSPACE
