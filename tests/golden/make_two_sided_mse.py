"""Write two_sided_lowbit_mse.json: the reconstruction MSE of the oracle's own
two-sided round trip on the seeded 8192 x 8192 bf16 workload (outliers x100,
row and column Rademacher signs, groups of 64), for 2-bit and 3-bit codes.

Calls only the CPU oracle and the seeded input generators:
    python tests/golden/make_two_sided_mse.py
The round trip is the two-sided RHT (HARP explainer §5), the group quantizer,
dequantization and the inverse transform; MSE is the float64 mean of
(reconstruction - input)^2 over all elements, the input being the bf16 matrix
widened exactly.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from oracle import hadamard as oh  # noqa: E402
from oracle import quant as oq  # noqa: E402


def main() -> None:
    d = synth.two_sided_lowbit()
    xb = synth.bf16_bits_to_f32(d["x_bf16"]).astype(np.float64)
    y = oh.two_sided(xb, d["row_signs"], d["col_signs"])
    out = {"workload": "two_sided_lowbit 8192x8192 bf16, groups of 64", "mse": {}}
    for bits in (2, 3):
        r = oq.quantize(y, bits, 64)
        rec = oh.two_sided_inverse(oq.dequantize(r["u"], r["scales"], bits, 64), d["row_signs"], d["col_signs"])
        out["mse"][str(bits)] = float(((rec - xb) ** 2).mean())
    with open(os.path.join(HERE, "two_sided_lowbit_mse.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
