"""Bounded device-side waits report the waits that gave up (through the C ABI).

The wait is made to run out with the library's self-test kernel: one warp waits
on a shared-memory barrier that nothing completes, through the same
bounded-wait routine and counter as the persistent row kernels, so nothing is
in flight when it gives up and the context stays usable."""
import ctypes

import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from hadamard_incoherence_transforms_b200 import _lib
from oracle import hadamard as oh
from oracle import quant as oq
from tests._parity import check_quant, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu


def test_expired_wait_is_counted_and_reported():
    lib = hit.load()
    assert hit.wait_timeouts(reset=True) == 0
    hit.wait_selftest(1_000_000)  # gives up after 1 ms
    assert hit.wait_timeouts(reset=False) == 1
    # the C status: HIT_ETIMEOUT with the count, and the reset clears it
    n = ctypes.c_ulonglong(0)
    assert lib.hit_wait_timeouts(ctypes.byref(n), 1) == _lib.HIT_ETIMEOUT
    assert n.value == 1
    assert b"gave up" in lib.hit_last_error()
    n = ctypes.c_ulonglong(0)
    assert lib.hit_wait_timeouts(ctypes.byref(n), 1) == _lib.HIT_OK and n.value == 0
    # two more on a side stream add up
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        hit.wait_selftest(2000)
        hit.wait_selftest(2000)
    assert hit.wait_timeouts(reset=True) == 2


def test_context_usable_after_expired_wait():
    hit.wait_selftest(1000)
    assert hit.wait_timeouts(reset=True) == 1
    d = synth.weight_rht_int4(rows=300, n=4096, seed=5)
    codes, scales = hit.rht_quantize_pack(to_gpu_f32(d["x"]), to_gpu_i8(d["signs"]), 4, 128)
    torch.cuda.synchronize()
    check_quant(codes, scales, oq.quantize(oh.rht_rows(d["x"], d["signs"]), 4, 128), 4, 4096)
    assert hit.wait_timeouts(reset=True) == 0
