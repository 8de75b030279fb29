"""B200-native batched randomized Walsh-Hadamard transforms for incoherence
processing: row / column RHT, mixed-radix stride butterflies, fused group
quantization with code packing, dequantize + inverse, and the sparse WHT
adapter expansion.  The work runs in libhit.so (CUDA, sm_100a) behind the C
ABI in include/hit.h; this package is a thin PyTorch binding over it.
"""
from ._lib import HitError, LIB_PATH, load  # noqa: F401
from .api import (  # noqa: F401
    butterfly_apply,
    butterfly_apply_tc,
    butterfly_tc_workspace_bytes,
    codes_shape,
    dequant_inverse,
    harp_blocks,
    harp_n_params,
    qwha_allocate,
    qwha_select,
    rht_forward,
    rht_inverse,
    rht_mixed_quantize_pack,
    rht_quantize_pack,
    row_norms,
    wait_selftest,
    wait_timeouts,
    wht_expand,
    wht_expand_2d,
    wht_gather,
    wht_gather_2d,
    workspace_bytes,
)

__version__ = "0.1.0"
