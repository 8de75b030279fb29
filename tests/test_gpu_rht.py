"""GPU parity of rht_forward / rht_inverse (through the C ABI) against the oracle."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import hadamard as oh
from tests._parity import assert_close, host, to_gpu_bf16, to_gpu_f32, to_gpu_i8

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def make_input(rows, n, seed, dtype):
    rng = np.random.default_rng(seed)
    x = (rng.standard_t(3, size=(rows, n)) * 0.5).astype(np.float32)
    s = (rng.integers(0, 2, n, dtype=np.int8) * 2 - 1).astype(np.int8)
    if dtype == torch.bfloat16:
        bits = synth.to_bf16_bits(x)
        return to_gpu_bf16(bits), synth.bf16_bits_to_f32(bits), s
    return to_gpu_f32(x), x, s


def oracle_rows(x, s, inverse, cols=None):
    if cols is not None:
        assert not inverse
        return oh.rht_rows_at(x, s, cols)
    return oh.irht_rows(x, s) if inverse else oh.rht_rows(x, s)


@pytest.mark.parametrize("logn", list(range(0, 16)))
@pytest.mark.parametrize("dts", [("f32", "f32"), ("bf16", "bf16")])
def test_rows_forward_every_length(logn, dts):
    n = 1 << logn
    rows = {0: 300, 1: 257, 2: 129, 3: 131, 7: 130, 12: 7, 13: 5, 14: 3, 15: 3}.get(logn, 37)
    xin, x64, s = make_input(rows, n, 1000 + logn, DT[dts[0]])
    y = hit.rht_forward(xin, to_gpu_i8(s), out_dtype=DT[dts[1]])
    torch.cuda.synchronize()
    cols = None if n <= 8192 else np.unique(np.random.default_rng(logn).integers(0, n, 96))
    ref = oracle_rows(x64, s, False, cols)
    got = host(y) if cols is None else host(y)[:, cols]
    assert_close(got, ref, DT[dts[1]], f"n={n}")


@pytest.mark.parametrize("logn", [2, 5, 8, 9, 10, 11, 12, 13])
@pytest.mark.parametrize("dts", [("f32", "f32"), ("bf16", "bf16"), ("f32", "bf16"), ("bf16", "f32")])
def test_rows_inverse_and_dtypes(logn, dts):
    n = 1 << logn
    xin, x64, s = make_input(67, n, 2000 + logn, DT[dts[0]])
    y = hit.rht_inverse(xin, to_gpu_i8(s), out_dtype=DT[dts[1]])
    z = hit.rht_forward(xin, None, out_dtype=DT[dts[1]])
    torch.cuda.synchronize()
    assert_close(host(y), oh.irht_rows(x64, s), DT[dts[1]], "inverse")
    assert_close(host(z), oh.rht_rows(x64, None), DT[dts[1]], "no signs")


@pytest.mark.parametrize("logn", [4, 12])
def test_round_trip_in_place_and_padded_rows(logn):
    n = 1 << logn
    rng = np.random.default_rng(5)
    buf = torch.zeros((9, n + 64), dtype=torch.float32, device="cuda")
    x = rng.standard_normal((9, n)).astype(np.float32)
    view = buf[:, 16:16 + n]
    view.copy_(to_gpu_f32(x))
    s = to_gpu_i8((rng.integers(0, 2, n, dtype=np.int8) * 2 - 1).astype(np.int8))
    hit.rht_forward(view, s, out=view)  # in place, leading dimension n + 64
    torch.cuda.synchronize()
    assert_close(host(view), oh.rht_rows(x, s.cpu().numpy()), torch.float32, "in place")
    hit.rht_inverse(view, s, out=view)
    torch.cuda.synchronize()
    assert_close(host(view), x, torch.float32, "round trip")
    # padding columns untouched
    assert float(buf[:, :16].abs().max()) == 0.0 and float(buf[:, 16 + n:].abs().max()) == 0.0


@pytest.mark.parametrize("m", [1, 2, 8, 128, 256, 4096])
@pytest.mark.parametrize("dts", [("f32", "f32"), ("bf16", "bf16")])
def test_columns(m, dts):
    cols = 100
    xin, x64, _ = make_input(m, cols, 3000 + m, DT[dts[0]])
    s = (np.random.default_rng(m).integers(0, 2, m, dtype=np.int8) * 2 - 1).astype(np.int8)
    y = hit.rht_forward(xin, to_gpu_i8(s), axis=0, out_dtype=DT[dts[1]])
    yi = hit.rht_inverse(xin, to_gpu_i8(s), axis=0, out_dtype=DT[dts[1]])
    torch.cuda.synchronize()
    assert_close(host(y).T, oh.rht_cols(x64, s).T, DT[dts[1]], f"cols m={m}")
    assert_close(host(yi).T, oh.irht_cols(x64, s).T, DT[dts[1]], f"inverse cols m={m}")


def test_empty_rows_is_a_no_op():
    x = torch.empty((0, 64), dtype=torch.float32, device="cuda")
    y = hit.rht_forward(x)
    assert y.shape == (0, 64)


def test_activation_workload_full_size():
    """bf16 8192 x 4096 activations (Student-t, outlier columns), forward only,
    at the full size; every row checked on 64 sampled output columns."""
    d = synth.activation_rht()
    x = to_gpu_bf16(d["x_bf16"])
    y = hit.rht_forward(x, to_gpu_i8(d["signs"]))
    torch.cuda.synchronize()
    cols = np.unique(np.random.default_rng(2).integers(0, 4096, 64))
    x64 = synth.bf16_bits_to_f32(d["x_bf16"])
    ref = oh.rht_rows_at(x64, d["signs"], cols)
    assert_close(host(y)[:, cols], ref, torch.bfloat16, "activation workload")
    # full-row check of a few rows
    rows = np.array([0, 1, 4095, 8191])
    assert_close(host(y[rows.tolist()]), oh.rht_rows(x64[rows], d["signs"]), torch.bfloat16, "rows")


@pytest.mark.parametrize("m", [1024, 2048, 4096, 8192])
@pytest.mark.parametrize("cols", [32, 96])
@pytest.mark.parametrize("dts", [("f32", "f32"), ("bf16", "f32"), ("f32", "bf16")])
def test_columns_cluster_path(m, cols, dts):
    """Column lengths 1024..8192 with 32-column strips (the cluster kernel)."""
    xin, x64, _ = make_input(m, cols, 4000 + m + cols, DT[dts[0]])
    s = (np.random.default_rng(m + 1).integers(0, 2, m, dtype=np.int8) * 2 - 1).astype(np.int8)
    y = hit.rht_forward(xin, to_gpu_i8(s), axis=0, out_dtype=DT[dts[1]])
    yi = hit.rht_inverse(xin, to_gpu_i8(s), axis=0, out_dtype=DT[dts[1]])
    torch.cuda.synchronize()
    assert_close(host(y).T, oh.rht_cols(x64, s).T, DT[dts[1]], f"cluster cols m={m}")
    assert_close(host(yi).T, oh.irht_cols(x64, s).T, DT[dts[1]], f"cluster inverse cols m={m}")
