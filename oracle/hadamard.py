"""Dense Sylvester–Hadamard matrix and the randomized Hadamard rotation (oracle; test infrastructure only).

"Random-rotation quantization" page, section "Why rotation works": in practice
the rotation is the Randomized Hadamard Transform, computable in O(d log d) and
close enough to a uniform orthogonal transform.  "TurboQuant and per-layer
outlier-aware K" page, section "TurboQuant 2026": the rotation is the FWHT.

Reading (the pages fix neither ordering nor normalisation): H is Sylvester's
construction in natural order (H_1 = [1], H_2k = [[H, H], [H, -H]]), which is
the order an in-place FWHT produces; the rotation is Π = H·D/√d (signs first,
then the transform), orthogonal because H·Hᵀ = d·I.

The oracle uses the explicit dense matrix on purpose — no fast transform — so
it shares no structure with the GPU butterflies.

Pins: H·Hᵀ = d·I, equality with scipy's Hadamard construction, ‖Πx‖ = ‖x‖,
exact sign-enumeration moments of Πx (tests/test_oracle_pins.py).
"""

from __future__ import annotations

import numpy as np

from .rng import rotation_signs


def sylvester(d: int) -> np.ndarray:
    """Sylvester–Hadamard matrix of order d (a power of two), float64, entries +-1."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_matrix(seed: int, d: int) -> np.ndarray:
    """Π = H·D/√d with D = diag(rotation_signs(seed, d))."""
    h = sylvester(d)
    s = rotation_signs(seed, d)
    return h * s[None, :] / np.sqrt(d)


def rotate(x: np.ndarray, seed: int, inverse: bool = False) -> np.ndarray:
    """Rows of x mapped by Π (or by Πᵀ when inverse), float64.  x: [..., d]."""
    x = np.asarray(x, dtype=np.float64)
    p = rotation_matrix(seed, x.shape[-1])
    return x @ (p if inverse else p.T)
