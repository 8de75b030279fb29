"""Pins for the oracle's mixed-radix butterfly (CPU only).

The reference evaluation here is a pure-Python loop over indices that spells
out the stage definition digit by digit; it shares nothing with the oracle's
einsum / moveaxis implementation.
"""
import itertools

import numpy as np
import pytest

from oracle import butterfly as ob
from synth import seeded_orthogonal_blocks
from tests.test_oracle_hadamard import popcount_hadamard


def loop_apply(x, radices, blocks, transpose=False):
    """Stage t: y[i] = sum_k B_{t,c}[i_t, k] x[i with digit t := k]; c = the other
    digits read as a row-major number; stages t = 0..m-1 (reversed and with
    transposed blocks for R^T)."""
    m = len(radices)
    d = int(np.prod(radices))
    x = [float(v) for v in x]
    order = list(range(m)) if not transpose else list(reversed(range(m)))
    for t in order:
        y = [0.0] * d
        for digits in itertools.product(*[range(b) for b in radices]):
            i = 0
            for b, dig in zip(radices, digits):
                i = i * b + dig
            c = 0
            for u, (b, dig) in enumerate(zip(radices, digits)):
                if u != t:
                    c = c * b + dig
            blk = blocks[t][0] if blocks[t].shape[0] == 1 else blocks[t][c]
            acc = 0.0
            for k in range(radices[t]):
                dk = list(digits)
                dk[t] = k
                j = 0
                for b, dig in zip(radices, dk):
                    j = j * b + dig
                coef = blk[k, digits[t]] if transpose else blk[digits[t], k]
                acc += float(coef) * x[j]
            y[i] = acc
        x = y
    return np.array(x)


def random_blocks(radices, shared=False, seed=0):
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    out = []
    for b in radices:
        g = 1 if shared else d // b
        out.append(rng.standard_normal((g, b, b)))  # general (not orthogonal) blocks
    return out


@pytest.mark.parametrize("radices", [(3, 4), (2, 3, 2), (5,), (4, 1, 3), (7, 2)])
@pytest.mark.parametrize("shared", [False, True])
@pytest.mark.parametrize("transpose", [False, True])
def test_matches_index_loop(radices, shared, transpose):
    blocks = random_blocks(radices, shared, seed=sum(radices))
    d = int(np.prod(radices))
    rng = np.random.default_rng(d)
    x = rng.standard_normal((3, d))
    got = ob.apply_stages(x, radices, blocks, transpose)
    for r in range(3):
        np.testing.assert_allclose(got[r], loop_apply(x[r], radices, blocks, transpose), atol=1e-12)


@pytest.mark.parametrize("radices", [(2, 2, 2), (4, 8), (16, 16), (8, 2, 4), (16, 16, 16)])
def test_all_hadamard_blocks_recover_hadamard(radices):
    d = int(np.prod(radices))
    blocks = [np.broadcast_to(popcount_hadamard(b) / np.sqrt(b), (d // b, b, b)) for b in radices]
    r = ob.dense(radices, blocks)
    np.testing.assert_allclose(r, popcount_hadamard(d) / np.sqrt(d), atol=1e-12)


def test_single_full_stage_is_matmul():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((1, 12, 12))
    x = rng.standard_normal((4, 12))
    np.testing.assert_allclose(ob.apply_stages(x, (12,), [a]), x @ a[0].T, atol=1e-12)
    np.testing.assert_allclose(ob.apply_stages(x, (12,), [a], transpose=True), x @ a[0], atol=1e-12)


@pytest.mark.parametrize("radices", [(7, 4, 2), (3, 5), (2, 7, 2, 2)])
def test_orthogonal_blocks_give_orthogonal_r(radices):
    rng = np.random.default_rng(11)
    d = int(np.prod(radices))
    blocks = [seeded_orthogonal_blocks(rng, d // b, b) for b in radices]
    r = ob.dense(radices, blocks)
    np.testing.assert_allclose(r.T @ r, np.eye(d), atol=1e-6)
    rt = ob.dense(radices, blocks, transpose=True)
    np.testing.assert_allclose(rt, r.T, atol=1e-12)


def test_full_schedule_norm_and_inverse():
    rng = np.random.default_rng(13)
    radices = (7, 16, 16, 8)
    d = 14336
    blocks = [seeded_orthogonal_blocks(rng, d // b, b).astype(np.float64) for b in radices]
    x = rng.standard_normal((3, d))
    y = ob.apply_stages(x, radices, blocks)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-5)
    np.testing.assert_allclose(ob.apply_stages(y, radices, blocks, transpose=True), x, atol=1e-5)


def test_columns_direction():
    rng = np.random.default_rng(17)
    radices = (3, 4)
    blocks = random_blocks(radices, seed=3)
    x = rng.standard_normal((12, 5))
    r = ob.dense(radices, blocks)
    np.testing.assert_allclose(ob.apply_stages_cols(x, radices, blocks), r @ x, atol=1e-12)


# --- mixed-radix randomized transform (signs, then the stage product) ---

def test_mixed_rht_equals_dense_sylvester_rht_for_power_of_two_radices():
    """With Hadamard blocks on every power-of-two radix the mixed-radix RHT is
    the RHT of the dense Sylvester path: (x * s) @ H_d / sqrt(d)."""
    rng = np.random.default_rng(5)
    radices = (4, 2, 8)
    d = 64
    x = rng.standard_normal((3, d))
    s = np.where(rng.random(d) < 0.5, -1, 1).astype(np.int8)
    y = ob.rht_mixed(x, s, radices, ob.rht_stage_blocks(radices))
    assert np.allclose(y, (x * s) @ popcount_hadamard(d) / 8.0, atol=1e-12)
    for b, blk in zip(radices, ob.rht_stage_blocks(radices)):
        assert np.array_equal(blk[0], popcount_hadamard(b) / np.sqrt(b))


def test_mixed_rht_with_radix_five_preserves_norms_and_inverts():
    rng = np.random.default_rng(6)
    radices = (8, 5, 2)
    d = 80
    blocks = ob.rht_stage_blocks(radices, {5: seeded_orthogonal_blocks(rng, d // 5, 5)})
    x = rng.standard_normal((4, d))
    s = np.where(rng.random(d) < 0.5, -1, 1).astype(np.int8)
    y = ob.rht_mixed(x, s, radices, blocks)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-6)
    assert np.allclose(ob.irht_mixed(y, s, radices, blocks), x, atol=1e-5)
    # the signs are applied before the stages: flipping s_j flips column j of R
    e = np.zeros((1, d))
    e[0, 7] = 1.0
    col = ob.rht_mixed(e, s, radices, blocks)[0]
    assert np.allclose(col, s[7] * ob.dense(radices, blocks)[:, 7], atol=1e-6)


def test_mixed_rht_synthetic_recipe():
    from synth import mixed_rht_int4

    d = mixed_rht_int4(rows=8)
    assert d["x"].shape == (8, 5120) and d["radices"] == (8, 8, 8, 5, 2)
    assert list(d["mixers"]) == [5] and d["mixers"][5].shape == (1, 5, 5)
    blocks = ob.rht_stage_blocks(d["radices"], d["mixers"])
    assert [b.shape for b in blocks] == [(1, 8, 8), (1, 8, 8), (1, 8, 8), (1, 5, 5), (1, 2, 2)]
    y = ob.rht_mixed(d["x"], d["signs"], d["radices"], blocks)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(d["x"].astype(np.float64), axis=1), rtol=1e-5)


@pytest.mark.parametrize("radices", [(8, 5, 2), (2, 3, 4), (5, 4), (3, 3, 2)])
def test_shared_blocks_give_the_kronecker_product(radices):
    """With one block per stage, R = B_0 (x) B_1 (x) ... (x) B_{m-1} (digit 0 most
    significant, the row-major convention of np.kron), so the order of the stages
    does not matter."""
    rng = np.random.default_rng(sum(radices))
    blocks = [rng.standard_normal((1, b, b)) for b in radices]
    want = blocks[0][0]
    for blk in blocks[1:]:
        want = np.kron(want, blk[0])
    np.testing.assert_allclose(ob.dense(radices, blocks), want, rtol=0, atol=1e-12)


def test_mixed_rht_is_harp_at_zero_parameters():
    """The mixed-radix RHT with one shared QR mixer is HARP's transform at theta = 0."""
    from oracle import harp as oha
    from synth import mixed_rht_int4

    d = mixed_rht_int4(rows=3, d=80, radices=(8, 5, 2))
    thetas = [np.zeros((80 // b, oha.n_params(b))) for b in d["radices"]]
    y_harp = oha.forward(d["x"], d["signs"], d["radices"], thetas, {5: d["mixers"][5][0]})
    y_rht = ob.rht_mixed(d["x"], d["signs"], d["radices"], ob.rht_stage_blocks(d["radices"], d["mixers"]))
    np.testing.assert_allclose(y_harp, y_rht, rtol=0, atol=1e-14)
