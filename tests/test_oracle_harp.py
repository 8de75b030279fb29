"""Pins for the oracle's HARP blocks B(theta) = Q(theta) G (CPU only).

The expected values come from closed forms worked out by hand: a Cayley map
whose skew matrix lives in one coordinate plane is the plane rotation with
cos = (1 - a^2) / (1 + a^2) and sin = 2a / (1 + a^2); skew matrices on disjoint
planes give a direct sum; the Cayley map is I + 2A to first order and
Q(-theta) = Q(theta)^T; at theta = 0 the blocks are the fixed mixers and the
transform is the popcount Sylvester RHT.  Each pin is written as a predicate
over the functions under test so that planted mistakes can be shown to fail.
"""
import numpy as np
import pytest

from oracle import harp as oha
from tests.test_oracle_butterfly import loop_apply
from tests.test_oracle_hadamard import popcount_hadamard

# Strict upper-triangle pairs of a 4 x 4 matrix in parameter order (row by row), written out.
PAIRS4 = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]


def plane_rotation(b, i, j, a):
    """Closed form of (I - A)^-1 (I + A) for A = a (e_i e_j^T - e_j e_i^T)."""
    q = np.eye(b)
    den = 1.0 + a * a
    q[i, i] = q[j, j] = (1.0 - a * a) / den
    q[i, j] = 2.0 * a / den
    q[j, i] = -2.0 * a / den
    return q


def cayley_plane_pin(cayley):
    for k, (i, j) in enumerate(PAIRS4):
        for a in (0.25, -1.5, 3.0):
            th = np.zeros(6)
            th[k] = a
            if not np.allclose(cayley(th, 4), plane_rotation(4, i, j, a), rtol=0, atol=1e-14):
                return False
    return True


def cayley_direct_sum_pin(cayley):
    th = np.zeros(6)
    th[0], th[5] = 0.5, -2.0          # planes (0,1) and (2,3)
    want = plane_rotation(4, 0, 1, 0.5) @ plane_rotation(4, 2, 3, -2.0)
    return np.allclose(cayley(th, 4), want, rtol=0, atol=1e-14)


def cayley_first_order_pin(cayley):
    rng = np.random.default_rng(11)
    for b in (3, 5, 8):
        m = b * (b - 1) // 2
        th = rng.standard_normal(m)
        a = np.zeros((b, b))
        k = 0
        for i in range(b):
            for j in range(i + 1, b):
                a[i, j], a[j, i] = th[k], -th[k]
                k += 1
        eps = 1e-7
        if not np.allclose((cayley(eps * th, b) - np.eye(b)) / eps, 2.0 * a, rtol=0, atol=1e-5):
            return False
    return True


def test_cayley_single_parameter_is_the_plane_rotation():
    assert cayley_plane_pin(oha.cayley)


def test_cayley_disjoint_planes_give_a_direct_sum():
    assert cayley_direct_sum_pin(oha.cayley)


def test_cayley_first_order_is_identity_plus_twice_the_skew_matrix():
    assert cayley_first_order_pin(oha.cayley)


@pytest.mark.parametrize("b", [3, 4, 5, 7, 8, 16])
def test_cayley_orthogonal_det_one_and_inverse_by_negation(b):
    rng = np.random.default_rng(b)
    th = rng.standard_normal(b * (b - 1) // 2) * 0.7
    q = oha.cayley(th, b)
    np.testing.assert_allclose(q.T @ q, np.eye(b), rtol=0, atol=1e-12)
    assert abs(np.linalg.det(q) - 1.0) < 1e-12
    np.testing.assert_allclose(oha.cayley(-th, b), q.T, rtol=0, atol=1e-12)


def test_cayley_half_turn_at_unit_parameter():
    # a = 1 in one plane: cos = 0, sin = 1, an exact quarter turn.
    want = np.array([[0.0, 1.0, 0.0], [-1.0, 0.0, 0.0], [0.0, 0.0, 1.0]])
    np.testing.assert_array_equal(np.round(oha.cayley([1.0, 0.0, 0.0], 3), 15), want)


def test_givens_entries_and_cayley_relation():
    phi = 0.3
    c, s = np.cos(phi), np.sin(phi)
    np.testing.assert_array_equal(oha.givens(phi), np.array([[c, -s], [s, c]]))
    # A 2 x 2 Cayley map of parameter a is the rotation by -2 atan(a).
    for a in (0.1, -0.7, 2.0):
        np.testing.assert_allclose(oha.cayley([a], 2), oha.givens(-2.0 * np.arctan(a)), rtol=0, atol=1e-15)


def radix2_block_pin(blocks_fn):
    """b = 2, G = H_2 / sqrt 2: B(phi) = [[c - s, c + s], [s + c, s - c]] / sqrt 2."""
    phis = np.array([[0.2], [-1.1]])
    got = blocks_fn([phis, np.zeros((2, 1))], (2, 2))[0]
    for c_, phi in enumerate(phis[:, 0]):
        c, s = np.cos(phi), np.sin(phi)
        want = np.array([[c - s, c + s], [s + c, s - c]]) / np.sqrt(2.0)
        if not np.allclose(got[c_], want, rtol=0, atol=1e-15):
            return False
    return True


def test_radix2_block_is_rotation_times_hadamard():
    assert radix2_block_pin(oha.blocks)


@pytest.mark.parametrize("radices", [(2, 4), (4, 2, 2), (16,), (8, 8)])
def test_zero_parameters_give_the_sylvester_rht(radices):
    d = int(np.prod(radices))
    thetas = [np.zeros((d // b, oha.n_params(b))) for b in radices]
    rng = np.random.default_rng(d)
    x = rng.standard_normal((3, d))
    s = rng.choice([-1.0, 1.0], size=d)
    want = (x * s) @ popcount_hadamard(d) / np.sqrt(d)
    np.testing.assert_allclose(oha.forward(x, s, radices, thetas), want, rtol=0, atol=1e-12)


def test_zero_parameters_keep_the_qr_mixer():
    rng = np.random.default_rng(5)
    g5, _ = np.linalg.qr(rng.standard_normal((5, 5)))
    thetas = [np.zeros((10 // 2, 1)), np.zeros((10 // 5, 10))]
    blk = oha.blocks(thetas, (2, 5), {5: g5})
    for c in range(2):
        np.testing.assert_array_equal(blk[1][c], g5)
    np.testing.assert_allclose(blk[0][0], popcount_hadamard(2) / np.sqrt(2.0), rtol=0, atol=1e-16)


@pytest.mark.parametrize("radices", [(2, 3), (4, 5), (3, 2, 2)])
def test_transform_matches_index_loop_and_is_orthogonal(radices):
    rng = np.random.default_rng(sum(radices))
    d = int(np.prod(radices))
    mixers = {b: np.linalg.qr(rng.standard_normal((b, b)))[0] for b in radices if b & (b - 1)}
    thetas = [rng.standard_normal((d // b, oha.n_params(b))) * 0.3 for b in radices]
    blk = oha.blocks(thetas, radices, mixers)
    s = rng.choice([-1.0, 1.0], size=d)
    x = rng.standard_normal(d)
    want = loop_apply(x * s, radices, blk)
    np.testing.assert_allclose(oha.forward(x[None], s, radices, thetas, mixers)[0], want, rtol=0, atol=1e-12)
    r = oha.forward(np.eye(d), s, radices, thetas, mixers)
    np.testing.assert_allclose(r @ r.T, np.eye(d), rtol=0, atol=1e-12)
    back = oha.inverse(oha.forward(x[None], s, radices, thetas, mixers), s, radices, thetas, mixers)
    np.testing.assert_allclose(back[0], x, rtol=0, atol=1e-12)


def test_parameter_counts_and_shape_checks():
    assert [oha.n_params(b) for b in (1, 2, 3, 5, 8, 16)] == [0, 1, 3, 10, 28, 120]
    with pytest.raises(ValueError):
        oha.blocks([np.zeros((4, 2))], (4,))          # wrong parameter count
    with pytest.raises(ValueError):
        oha.blocks([np.zeros((1, 10))], (5,))         # no mixer for radix 5


def int8_pin(to_int8):
    """max |theta| = 127 gives scale 1 exactly, so q is rint(theta) with ties to even."""
    q, scale = to_int8(np.array([127.0, 2.5, -3.5, 0.49, -127.0, 126.5], np.float32))
    return scale == np.float32(1.0) and q.tolist() == [127, 2, -4, 0, -127, 126]


def test_int8_hand_cases():
    assert int8_pin(oha.theta_to_int8)
    q, scale = oha.theta_to_int8(np.zeros(7))
    assert scale == 0 and not q.any()
    assert not oha.theta_from_int8(q, scale).any()


def test_int8_error_bound_and_extremes():
    rng = np.random.default_rng(3)
    th = (rng.standard_normal(1000) * 0.05).astype(np.float32)
    q, scale = oha.theta_to_int8(th)
    assert scale == np.float32(np.max(np.abs(th)) / np.float32(127))
    assert np.abs(q).max() == 127 and q[np.argmax(np.abs(th))] == np.sign(th[np.argmax(np.abs(th))]) * 127
    back = oha.theta_from_int8(q, scale)
    assert np.all(np.abs(back.astype(np.float64) - th) <= scale * (0.5 + 1e-6))


def test_int8_parameters_keep_the_transform_orthogonal():
    rng = np.random.default_rng(9)
    radices = (4, 4)
    thetas = [rng.standard_normal((4, 6)) * 0.2 for _ in radices]
    stored = [oha.theta_from_int8(*oha.theta_to_int8(t)) for t in thetas]
    r = oha.forward(np.eye(16), np.ones(16), radices, stored)
    np.testing.assert_allclose(r @ r.T, np.eye(16), rtol=0, atol=1e-12)


def test_pins_reject_planted_mistakes():
    def cayley_swapped(th, b):             # (I + A)^-1 (I - A): the transpose
        return oha.cayley(th, b).T

    def cayley_col_major(th, b):           # parameters down the columns instead of along the rows
        a = np.zeros((b, b))
        k = 0
        for j in range(b):
            for i in range(j):
                a[i, j], a[j, i] = th[k], -th[k]
                k += 1
        return np.linalg.solve(np.eye(b) - a, np.eye(b) + a)

    def cayley_half(th, b):                # exponential-like map with half the angle
        return oha.cayley(np.asarray(th) / 2.0, b)

    for bad in (cayley_swapped, cayley_col_major, cayley_half):
        assert not (cayley_plane_pin(bad) and cayley_direct_sum_pin(bad) and cayley_first_order_pin(bad))

    def blocks_mixer_first(thetas, radices, mixers=None):   # G Q instead of Q G
        out = []
        for t, b in enumerate(radices):
            g = oha.base_mixer(b, (mixers or {}).get(b))
            out.append(np.stack([g @ oha.learnable_factor(th, b) for th in thetas[t]]))
        return out

    assert not radix2_block_pin(blocks_mixer_first)

    def int8_floor(theta):
        th = np.asarray(theta, np.float32)
        scale = np.float32(np.max(np.abs(th)) / np.float32(127))
        return np.floor(th / scale + np.float32(0.5)).astype(np.int8), scale

    assert not int8_pin(int8_floor)
