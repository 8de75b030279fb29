"""Readers for the hand-worked fixtures under tests/golden/."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield [p.strip() for p in line.split("|")]


def _vec(text):
    scale = 1.0
    if text.startswith("r2*"):
        scale, text = 1.0 / np.sqrt(2.0), text[3:]
    return np.array([float(v) for v in text.split(",")], dtype=np.float64) * scale


def rht_cases():
    for n, x, s, y in _rows("rht_hand_examples.txt"):
        yield int(n), _vec(x), _vec(s), _vec(y)


def quant_cases():
    for bits, y, scale, q, packed, yhat in _rows("quant_hand_examples.txt"):
        yield (int(bits), np.array([float(v) for v in y.split(",")], np.float32), np.float32(scale),
               np.array([int(v) for v in q.split(",")]), bytes(int(b, 16) for b in packed.split(",")),
               np.array([float(v) for v in yhat.split(",")], np.float32))
