"""The seeded input generators follow their recipes (CPU only)."""
import numpy as np
import torch

import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0], np.float32)])
    bits = synth.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.uint16).numpy()
    assert np.array_equal(bits, ref)
    assert np.array_equal(synth.bf16_bits_to_f32(bits), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_weight_recipe_small():
    a = synth.weight_rht_int4(rows=64, n=256)
    b = synth.weight_rht_int4(rows=64, n=256)
    assert np.array_equal(a["x"], b["x"]) and np.array_equal(a["signs"], b["signs"])
    assert a["x"].dtype == np.float32 and a["x"].shape == (64, 256)
    assert len(a["outliers"]) == round(0.001 * 64 * 256) == len(np.unique(a["outliers"]))
    assert set(np.unique(a["signs"])) <= {-1, 1}


def test_sparse_columns_distinct_and_sorted():
    rng = np.random.default_rng(4)
    cols = synth.sparse_columns(rng, 2000, 4096, 64)
    assert cols.dtype == np.int32 and cols.shape == (2000, 64)
    assert np.all(np.diff(cols, axis=1) > 0)
    assert cols.min() >= 0 and cols.max() < 4096


def test_orthogonal_blocks():
    rng = np.random.default_rng(5)
    q = synth.seeded_orthogonal_blocks(rng, 10, 7).astype(np.float64)
    np.testing.assert_allclose(np.einsum("gij,gik->gjk", q, q), np.broadcast_to(np.eye(7), (10, 7, 7)), atol=1e-6)


def test_two_sided_recipe_small():
    d = synth.two_sided_lowbit(rows=64, n=128)
    assert d["x_bf16"].dtype == np.uint16 and d["x_bf16"].shape == (64, 128)
    assert d["row_signs"].shape == (128,) and d["col_signs"].shape == (64,)


def test_harp_recipe_small():
    a = synth.harp_rotation(rows=8, d=64, radices=(4, 4, 4))
    b = synth.harp_rotation(rows=8, d=64, radices=(4, 4, 4))
    assert all(np.array_equal(p, q) for p, q in zip(a["thetas"], b["thetas"]))
    assert [t.shape for t in a["thetas"]] == [(16, 6)] * 3 and a["base_mixers"] == {}
    c = synth.harp_rotation(rows=8, d=80, radices=(8, 5, 2))
    assert [t.shape for t in c["thetas"]] == [(10, 28), (16, 10), (40, 1)]
    g = c["base_mixers"][5].astype(np.float64)
    np.testing.assert_allclose(g.T @ g, np.eye(5), atol=1e-6)
    assert abs(float(np.std(np.concatenate([t.ravel() for t in c["thetas"]]))) - 0.05) < 0.01


def test_qwha_recipe_small():
    d = synth.qwha_init(rows=32, n=128, tokens=16, per_row=8)
    assert d["w"].shape == (32, 128) and d["x"].shape == (128, 16) and d["budget"] == 256
    assert len(d["outlier_channels"]) == round(0.01 * 128)
    assert np.all(np.abs(d["x"][d["outlier_channels"]]).mean(axis=1) > 5)
