"""ctypes loader for libhit.so and the raw C entry points (same names as hit.h).

The library is built in-tree by ``python -m hadamard_incoherence_transforms_b200.build``
(or ``__graft_entry__.build()``).  Loading fails loudly if it is missing: there
is no other implementation of these operations in this package.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhit.so")

HIT_OK, HIT_EINVAL, HIT_EUNSUPPORTED, HIT_EALIGN, HIT_ECUDA, HIT_EWORKSPACE, HIT_ETIMEOUT = 0, -1, -2, -3, -4, -5, -6
HIT_F32, HIT_BF16 = 0, 1
HIT_OP_RHT, HIT_OP_QUANT, HIT_OP_DEQUANT, HIT_OP_BUTTERFLY = 0, 1, 2, 3

_i64, _i32, _vp, _sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t

# name -> (restype, argtypes), in the order of include/hit.h
SIGNATURES = {
    "hit_version": (_i32, []),
    "hit_status_string": (ctypes.c_char_p, [_i32]),
    "hit_last_error": (ctypes.c_char_p, []),
    "hit_workspace_bytes": (_sz, [_i32, _i64, _i64, _i32, _i32]),
    "hit_wait_timeouts": (_i32, [ctypes.POINTER(ctypes.c_ulonglong), _i32]),
    "hit_wait_selftest": (_i32, [_i64, _vp]),
    "rht_forward": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "rht_inverse": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32, _vp, _i32, _vp, _sz, _vp]),
    "butterfly_apply": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _i32,
                               _vp, _sz, _vp]),
    "butterfly_apply_tc": (_i32, [_vp, _vp, _i64, _i64, _i64, _i64, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _i32,
                                  _vp, _sz, _vp]),
    "butterfly_tc_workspace_bytes": (_sz, [_i64, _i64, _i32, _i32, _vp, _i32]),
    "rht_quantize_pack": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _sz, _vp]),
    "rht_mixed_quantize_pack": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _i32, _i32, _vp, _vp, _vp]),
    "dequant_inverse": (_i32, [_vp, _vp, _i64, _i64, _i32, _i32, _vp, _vp, _vp, _i64, _i32, _vp, _sz, _vp]),
    "wht_expand_sparse": (_i32, [_vp, _vp, _i64, _i64, _i64, _i32, ctypes.c_float, _vp, _i32, _vp]),
    "wht_expand_sparse_2d": (_i32, [_vp, _vp, _i64, _i64, _i64, _i32, ctypes.c_float, _vp, _i32, _vp, _sz, _vp]),
    "row_norms": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp]),
    "qwha_allocate": (_i32, [_vp, _i64, _i64, _i64, _i64, _vp]),
    "qwha_select": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "harp_blocks": (_i32, [_vp, _vp, ctypes.c_float, _i64, _i32, _vp, _vp, _vp, _vp]),
    "rht_quantize_pack_noalloc": (_i32, [_vp, _i64, _i64, _i64, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp]),
}

_lib = None


class HitError(RuntimeError):
    """A libhit call returned a non-zero status."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status}: {msg}")
        self.status = status


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing; build it with `python -m hadamard_incoherence_transforms_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def call(name: str, *args) -> None:
    """Call a C entry point and raise HitError on a non-zero status."""
    lib = load()
    status = getattr(lib, name)(*args)
    if status != HIT_OK:
        raise HitError(name, status, lib.hit_last_error().decode(errors="replace"))
