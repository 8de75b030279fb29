"""HARP's parameterised stage blocks B_{t,c}(theta) = Q_{t,c}(theta) G_{b_t},
in float64 (test oracle only).

HARP explainer, technical summary §2.2: each learnable block is a learnable
orthogonal factor Q_{t,c}(theta) times a fixed base mixer G_{b_t}; the mixer is
the normalized Sylvester Hadamard for power-of-two radices and a deterministic
orthogonal substitute (QR of a fixed Gaussian) otherwise; Q is a Givens
rotation for b_t = 2 and a Cayley map for b_t > 2; all parameters start at
zero, where Q = I and the processor is exactly the fixed RHT.  §2.4: the
parameters can be stored as int8.

Readings taken where the pages stop:

* Givens, b = 2, one angle phi per block:
  Q = [[cos phi, -sin phi], [sin phi, cos phi]].
* Cayley, b > 2, b (b - 1) / 2 parameters per block: A is skew-symmetric with
  A[i, j] = theta_k and A[j, i] = -theta_k, where k enumerates the pairs i < j
  row by row ((0,1), (0,2), ..., (0,b-1), (1,2), ...); Q = (I - A)^-1 (I + A).
  b = 1 has no parameters and Q = [1].
* One base mixer per radix value, shared by every stage and group with that
  radix (the pages write G_{b_t}, indexed by the radix alone); the QR mixer of
  a non-power-of-two radix is an input (drawn by the seeded generators).
* The full HARP transform keeps the RHT's sign diagonal: y = R(theta) diag(s) x
  with R(theta) = B_{m-1} ... B_0 applied by the mixed-radix stage convention of
  :mod:`oracle.butterfly`; at theta = 0 and power-of-two radices this is the
  Sylvester RHT H_d diag(s) / sqrt(d).
* int8 storage: per stage, symmetric absmax with one fp32 scale,
  scale = max |theta| / 127 (correctly rounded), q = rint(theta / scale) with
  ties to even, clamped to [-127, 127]; an all-zero stage stores scale 0 and
  q = 0; the stored parameters are fp32(q) * scale.

Pinned by tests/test_oracle_harp.py: the Cayley map of a single parameter
against the closed-form plane rotation (pair order and sign), the two-parameter
disjoint-plane case against a direct sum, the first-order expansion
Q ~ I + 2A, Q(-theta) = Q(theta)^T, orthogonality and det = +1, the b = 2
Cayley/Givens relation phi = -2 atan(theta), the b = 2 block Q G written out
entry by entry, theta = 0 against the popcount Hadamard, and hand-worked int8
cases.
"""
from __future__ import annotations

import numpy as np

from .butterfly import apply_stages
from .hadamard import is_pow2, sylvester


def n_params(b: int) -> int:
    """Learnable parameters per b x b block: 0 (b = 1), 1 (Givens), b(b-1)/2 (Cayley)."""
    b = int(b)
    if b < 1:
        raise ValueError("radix must be >= 1")
    return 0 if b == 1 else 1 if b == 2 else b * (b - 1) // 2


def skew(theta, b: int) -> np.ndarray:
    """The b x b skew-symmetric A with the parameters on the strict upper triangle, row by row."""
    theta = np.asarray(theta, dtype=np.float64)
    if theta.shape != (b * (b - 1) // 2,):
        raise ValueError(f"a {b}x{b} skew matrix takes {b * (b - 1) // 2} parameters")
    a = np.zeros((b, b), dtype=np.float64)
    k = 0
    for i in range(b):
        for j in range(i + 1, b):
            a[i, j] = theta[k]
            a[j, i] = -theta[k]
            k += 1
    return a


def cayley(theta, b: int) -> np.ndarray:
    """Q = (I - A)^-1 (I + A) for A = skew(theta, b); I - A is always invertible
    (the eigenvalues of a real skew matrix are imaginary)."""
    a = skew(theta, b)
    eye = np.eye(b)
    return np.linalg.solve(eye - a, eye + a)


def givens(phi: float) -> np.ndarray:
    """The 2 x 2 rotation by angle phi."""
    c, s = np.cos(phi), np.sin(phi)
    return np.array([[c, -s], [s, c]], dtype=np.float64)


def learnable_factor(theta, b: int) -> np.ndarray:
    """Q(theta) for one b x b block: Givens for b = 2, Cayley for b > 2, [1] for b = 1."""
    theta = np.asarray(theta, dtype=np.float64).reshape(-1)
    if theta.size != n_params(b):
        raise ValueError(f"radix {b} takes {n_params(b)} parameters, got {theta.size}")
    if b == 1:
        return np.ones((1, 1))
    if b == 2:
        return givens(float(theta[0]))
    return cayley(theta, b)


def base_mixer(b: int, fallback=None) -> np.ndarray:
    """G_b: H_b / sqrt(b) for a power of two, else the given orthogonal b x b matrix."""
    if is_pow2(b):
        return sylvester(b) / np.sqrt(b)
    if fallback is None:
        raise ValueError(f"radix {b} is not a power of two: its orthogonal mixer must be given")
    g = np.asarray(fallback, dtype=np.float64)
    if g.shape != (b, b):
        raise ValueError(f"mixer for radix {b} must be {b}x{b}")
    return g


def blocks(thetas, radices, base_mixers=None) -> list[np.ndarray]:
    """Per stage t the [d / b_t, b_t, b_t] blocks B_{t,c} = Q(thetas[t][c]) G_{b_t}.

    thetas[t]: [d / b_t, n_params(b_t)]; base_mixers: {radix: b x b orthogonal}
    for the radices that are not powers of two.
    """
    radices = [int(b) for b in radices]
    d = int(np.prod(radices))
    mixers = base_mixers or {}
    out = []
    for t, b in enumerate(radices):
        th = np.asarray(thetas[t], dtype=np.float64)
        if th.shape != (d // b, n_params(b)):
            raise ValueError(f"stage {t}: thetas must be [{d // b}, {n_params(b)}]")
        g = base_mixer(b, mixers.get(b))
        out.append(np.stack([learnable_factor(th[c], b) @ g for c in range(d // b)]))
    return out


def forward(x, signs, radices, thetas, base_mixers=None) -> np.ndarray:
    """y = R(theta) diag(s) x for every row of x."""
    x = np.asarray(x, dtype=np.float64) * np.asarray(signs, dtype=np.float64)
    return apply_stages(x, radices, blocks(thetas, radices, base_mixers))


def inverse(y, signs, radices, thetas, base_mixers=None) -> np.ndarray:
    """x = diag(s) R(theta)^T y for every row of y."""
    out = apply_stages(y, radices, blocks(thetas, radices, base_mixers), transpose=True)
    return out * np.asarray(signs, dtype=np.float64)


def theta_to_int8(theta) -> tuple[np.ndarray, np.float32]:
    """Symmetric absmax int8 storage of one stage's parameters: (q, scale)."""
    th = np.asarray(theta).astype(np.float32)
    a = np.float32(np.max(np.abs(th))) if th.size else np.float32(0.0)
    scale = np.float32(a / np.float32(127.0))
    if scale == 0:
        return np.zeros(th.shape, dtype=np.int8), np.float32(0.0)
    q = np.clip(np.rint((th / scale).astype(np.float32)), -127, 127).astype(np.int8)
    return q, scale


def theta_from_int8(q, scale) -> np.ndarray:
    """Stored parameters fp32(q) * scale."""
    return (np.asarray(q, dtype=np.int8).astype(np.float32) * np.float32(scale)).astype(np.float32)
