"""The pins catch plausible oracle mistakes (CPU only).

Each test plants a mistake in a copy of an oracle function -- a dropped
normalisation, signs applied on the wrong side, a transposed block, floor in
place of rint, nibbles in the wrong order -- and checks that the pin it should
trip actually fails.  The real oracle passes the same checks in the other test
modules.
"""
import numpy as np

from oracle import hadamard as oh
from oracle import quant as oq
from oracle import butterfly as ob
from tests._golden import quant_cases, rht_cases
from tests.test_oracle_butterfly import loop_apply, random_blocks


def rht_pins_hold(fwd):
    for n, x, s, y in rht_cases():
        if not np.allclose(fwd(x[None, :], s)[0], y, atol=1e-12):
            return False
    return True


def test_rht_pins_reject_mutants():
    assert rht_pins_hold(oh.rht_rows)

    def no_norm(x, s):
        return (np.asarray(x) * s) @ oh.sylvester(x.shape[-1])

    def signs_after(x, s):
        return ((np.asarray(x) @ oh.sylvester(x.shape[-1])) / np.sqrt(x.shape[-1])) * s

    def wrong_recursion(x, s):
        n = x.shape[-1]
        h = oh.sylvester(n)
        if n >= 2:
            h = h[::-1]
        return ((np.asarray(x) * s) @ h) / np.sqrt(n)

    for mutant in (no_norm, signs_after, wrong_recursion):
        assert not rht_pins_hold(mutant)


def quant_pins_hold(quantize, pack):
    for bits, y, scale, q, packed, yhat in quant_cases():
        r = quantize(y[None, :], bits, 4)
        if r["scales"][0, 0] != scale or not np.array_equal(r["q"][0], q):
            return False
        if bytes(pack(r["u"], bits)[0]) != packed:
            return False
    return True


def test_quant_pins_reject_mutants():
    assert quant_pins_hold(oq.quantize, oq.pack)

    def floor_quant(y, bits, group):
        r = oq.quantize(y, bits, group)
        qm = (1 << (bits - 1)) - 1
        q = np.clip(np.floor(r["t"] + 0.5), -qm, qm).astype(np.int8)   # ties away from even
        r["q"] = q
        r["u"] = (q.astype(np.int16) + (1 << (bits - 1))).astype(np.uint8)
        return r

    def asym_scale(y, bits, group):
        r = oq.quantize(y, bits, group)
        r["scales"] = (r["scales"] * np.float32((1 << (bits - 1)) - 1) / np.float32(1 << (bits - 1))).astype(np.float32)
        return r

    def msb_first(u, bits):
        u = np.asarray(u, np.uint8)
        rows, n = u.shape
        st = ((u[..., None] >> np.arange(bits, dtype=np.uint8)) & 1).reshape(rows, n * bits)
        return np.packbits(st, axis=-1, bitorder="big")

    assert not quant_pins_hold(floor_quant, oq.pack)
    assert not quant_pins_hold(asym_scale, oq.pack)
    assert not quant_pins_hold(oq.quantize, msb_first)


def test_butterfly_pins_reject_transposed_blocks():
    radices = (3, 4)
    blocks = random_blocks(radices, seed=9)
    x = np.random.default_rng(0).standard_normal((1, 12))
    ref = loop_apply(x[0], radices, blocks)
    assert np.allclose(ob.apply_stages(x, radices, blocks)[0], ref, atol=1e-12)
    flipped = [np.swapaxes(b, -1, -2) for b in blocks]
    assert not np.allclose(ob.apply_stages(x, radices, flipped)[0], ref, atol=1e-6)
    reversed_order = ob.apply_stages(x, radices[::-1], blocks[::-1])[0]
    assert not np.allclose(reversed_order, ref, atol=1e-6)
