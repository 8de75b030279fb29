"""GPU parity of wht_expand_sparse (forward expansion and backward gather)."""
import numpy as np
import pytest
import torch

import hadamard_incoherence_transforms_b200 as hit
import synth
from oracle import sparse as osp
from tests._parity import assert_close, host, to_gpu_f32

pytestmark = pytest.mark.gpu


def gpu_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("logn", [5, 6, 7, 8, 9, 10, 11, 12, 13])
def test_expand_and_gather_every_length(logn):
    n = 1 << logn
    nnz = min(64, n)
    d = synth.wht_adapter(batch=2, rows=max(3, 4096 // n) + 1, n=n, nnz=nnz, seed=logn)
    scale = 1.0 / np.sqrt(n)
    v, c = d["values"], d["cols"]
    dense = hit.wht_expand(to_gpu_f32(v), gpu_i32(c), n, scale)
    g = synth.dense_gradient(*dense.shape, seed=logn)
    gv = hit.wht_gather(to_gpu_f32(g), gpu_i32(c), scale)
    torch.cuda.synchronize()
    assert_close(host(dense), osp.expand(v, c, n, scale), torch.float32, "expand")
    assert_close(host(gv), osp.gather_grad(g, c, scale), torch.float32, "gather")


def test_duplicates_and_out_of_range_columns():
    n = 256
    v = np.array([[[1.0, 2.0, -0.5, 7.0]]], np.float32)
    c = np.array([[[3, 3, 9, 300]]], np.int32)  # 300 is out of range: ignored / gives 0
    dense = hit.wht_expand(to_gpu_f32(v), gpu_i32(c), n, 0.25)
    torch.cuda.synchronize()
    ok = c < n
    ref = osp.expand(np.where(ok, v, 0), np.where(ok, c, 0), n, 0.25)
    assert_close(host(dense), ref, torch.float32, "duplicates")
    g = np.random.default_rng(0).standard_normal((1, 1, n)).astype(np.float32)
    gv = host(hit.wht_gather(to_gpu_f32(g), gpu_i32(c), 0.25))
    torch.cuda.synchronize()
    ref_g = osp.gather_grad(g, np.where(ok, c, 0), 0.25)
    np.testing.assert_allclose(gv[ok], ref_g[ok], rtol=1e-5, atol=1e-6)
    assert gv[~ok][0] == 0.0


def test_adapter_workload_full_size():
    """32 x 4096 x 4096 expansion (64 nonzeros per row) and its backward at the
    full size; 48 rows of each batch element checked against the oracle."""
    d = synth.wht_adapter()
    scale = 1.0 / 64.0
    values, cols = to_gpu_f32(d["values"]), gpu_i32(d["cols"])
    dense = hit.wht_expand(values, cols, 4096, scale)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 2047, 4095] + list(range(200, 244)))
    for b in (0, 17, 31):
        ref = osp.expand(d["values"][b:b + 1, rows], d["cols"][b:b + 1, rows], 4096, scale)
        assert_close(host(dense[b, rows.tolist()]), ref[0], torch.float32, f"expand batch {b}")
    g = torch.randn(dense.shape, generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    gv = hit.wht_gather(g, cols, scale)
    torch.cuda.synchronize()
    for b in (0, 31):
        gh = host(g[b, rows.tolist()])[None]
        ref = osp.gather_grad(gh, d["cols"][b:b + 1, rows], scale)
        assert_close(host(gv[b, rows.tolist()]), ref[0], torch.float32, f"gather batch {b}")
