"""Property-based checks of the oracle (CPU only): invariants that hold for any
input, explored by hypothesis over shapes and values the fixed-seed pins do
not reach (subnormal and zero groups, odd radices, extreme budgets)."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import butterfly as ob
from oracle import harp as oha
from oracle import quant as oq
from oracle import qwha as oqw

SETTINGS = settings(max_examples=80, deadline=None)

f32_values = st.one_of(
    st.floats(min_value=-1e4, max_value=1e4, allow_nan=False, width=32),
    st.sampled_from([0.0, -0.0, 1e-40, -1e-40, 1.5, -2.5, 3.5]),   # zeros, subnormals, exact halves
)


@SETTINGS
@given(bits=st.sampled_from([2, 3, 4]), group=st.sampled_from([1, 2, 4, 8]), ngroups=st.integers(1, 6),
       data=st.data())
def test_quantizer_invariants(bits, group, ngroups, data):
    vals = data.draw(st.lists(f32_values, min_size=group * ngroups, max_size=group * ngroups))
    y = np.array(vals, dtype=np.float32)[None]
    r = oq.quantize(y, bits, group)
    qm = (1 << (bits - 1)) - 1
    q = r["q"][0].astype(np.int64)
    s = r["scales"][0].astype(np.float64)
    assert np.all(np.abs(q) <= qm)
    assert np.array_equal(r["u"][0], (q + (1 << (bits - 1))).astype(np.uint8))
    g = y[0].reshape(ngroups, group).astype(np.float64)
    for k in range(ngroups):
        a = np.max(np.abs(g[k]))
        if s[k] == 0:
            assert a == 0 or a / qm < 1e-45   # the scale underflows only for (sub)normal-tiny groups
            assert not q[k * group:(k + 1) * group].any()
            continue
        # the absmax element lands on +-qmax, and every element is within half a step (plus t's rounding)
        j = int(np.argmax(np.abs(g[k])))
        assert abs(q[k * group + j]) == qm
        err = np.abs(g[k] - q[k * group:(k + 1) * group] * s[k])
        assert np.all(err <= s[k] * (0.5 + 2.0 ** -20) + 1e-45)
    back = oq.dequantize(r["u"], r["scales"], bits, group)
    assert np.array_equal(back[0], (q.astype(np.float32) * np.repeat(r["scales"][0], group)).astype(np.float32))


@SETTINGS
@given(bits=st.sampled_from([2, 3, 4]), rows=st.integers(1, 3), n=st.integers(1, 70), data=st.data())
def test_pack_unpack_round_trip(bits, rows, n, data):
    u = np.array(data.draw(st.lists(st.integers(0, (1 << bits) - 1), min_size=rows * n, max_size=rows * n)),
                 dtype=np.uint8).reshape(rows, n)
    packed = oq.pack(u, bits)
    assert packed.shape == (rows, (n * bits + 7) // 8)
    assert np.array_equal(oq.unpack(packed, bits, n), u)
    # stream bit k of row 0 is bit (k mod 8) of byte k // 8, code j at bits [b j, b j + b)
    j = data.draw(st.integers(0, n - 1))
    got = sum(((int(packed[0, (bits * j + i) // 8]) >> ((bits * j + i) % 8)) & 1) << i for i in range(bits))
    assert got == u[0, j]


radix_lists = st.lists(st.integers(1, 7), min_size=1, max_size=4).filter(lambda r: int(np.prod(r)) <= 96)


@SETTINGS
@given(radices=radix_lists, shared=st.booleans(), seed=st.integers(0, 2 ** 32 - 1))
def test_butterfly_with_orthogonal_blocks_is_orthogonal(radices, shared, seed):
    rng = np.random.default_rng(seed)
    d = int(np.prod(radices))
    blocks = []
    for b in radices:
        cnt = 1 if shared else d // b
        q, _ = np.linalg.qr(rng.standard_normal((cnt, b, b)))
        blocks.append(q)
    r = ob.dense(radices, blocks)
    np.testing.assert_allclose(r.T @ r, np.eye(d), atol=1e-11)
    np.testing.assert_allclose(ob.dense(radices, blocks, transpose=True), r.T, atol=1e-12)


@SETTINGS
@given(b=st.integers(2, 12), scale=st.floats(1e-3, 10.0), seed=st.integers(0, 2 ** 32 - 1))
def test_harp_factor_is_a_rotation(b, scale, seed):
    rng = np.random.default_rng(seed)
    th = rng.standard_normal(oha.n_params(b)) * scale
    q = oha.learnable_factor(th, b)
    np.testing.assert_allclose(q.T @ q, np.eye(b), atol=1e-10)
    assert abs(np.linalg.det(q) - 1.0) < 1e-9


@SETTINGS
@given(rows=st.integers(1, 30), n=st.integers(1, 40), k_min=st.integers(0, 3), seed=st.integers(0, 2 ** 32 - 1),
       frac=st.floats(0.0, 1.0))
def test_allocation_invariants(rows, n, k_min, seed, frac):
    k_min = min(k_min, n)
    rng = np.random.default_rng(seed)
    e = np.abs(rng.standard_cauchy(rows)) * (rng.random(rows) < 0.8)   # heavy tails and exact zeros
    budget = rows * k_min + int(round(frac * rows * (n - k_min)))
    k = oqw.allocate(e, budget, k_min, n)
    assert k.sum() == budget and k.min() >= k_min and k.max() <= n
    for a in range(rows):
        for c in range(rows):
            if e[a] > e[c] and k[c] < n:
                assert k[a] >= k[c]
