"""B200-native batched randomized Walsh-Hadamard transforms for incoherence
processing: row / column RHT, mixed-radix stride butterflies, fused group
quantization with code packing, dequantize + inverse, and the sparse WHT
adapter expansion.  The work runs in libhit.so (CUDA, sm_100a) behind the C
ABI in include/hit.h; this package is a thin PyTorch binding over it.
"""
from ._lib import HitError, LIB_PATH, load  # noqa: F401
from .api import (  # noqa: F401
    butterfly_apply,
    codes_shape,
    dequant_inverse,
    rht_forward,
    rht_inverse,
    rht_quantize_pack,
    wait_selftest,
    wait_timeouts,
    wht_expand,
    wht_gather,
    workspace_bytes,
)

__version__ = "0.1.0"
