"""Lloyd–Max scalar codebook for N(0,1) (oracle; test infrastructure only).

"Random-rotation quantization" page, section "History", EDEN bullet: after
normalising the rotated vector so each coordinate is about N(0,1), quantise
with a Lloyd–Max codebook computed once for the standard normal; 1-bit levels
±√(2/π) ≈ ±0.798, 2-bit levels ±0.453, ±1.510.  Section "Three decoders, one
rotation", MSE decoder: each rotated coordinate goes to the nearest of the 2^b
centroids.

The pages give no iteration; this is Lloyd's alternation written out:
  thresholds τ_k = (c_k + c_{k+1}) / 2 (nearest-centroid cells), then
  centroids c_k = E[X | τ_{k-1} < X < τ_k] = (φ(τ_{k-1}) − φ(τ_k)) / (Φ(τ_k) − Φ(τ_{k-1}))
with τ_{-1} = −∞, τ_{L-1} = +∞, started from the N(0,1) quantiles of the cell
mid-probabilities and run until no level moves by more than 1e-14.

Distortion D_b = E[(X − Q(X))²] = 1 − Σ_k (φ(τ_{k-1}) − φ(τ_k))² / P_k at the
fixed point (centroid condition).

Pins: b=1 equals √(2/π) and D_1 = 1 − 2/π (closed form); b=2 rounds to the
page's ±0.453, ±1.510; b=3, 4 agree with Max (1960), Table I to the
precision printed there; symmetry; fixed-point residual
(tests/test_oracle_pins.py).
"""

from __future__ import annotations

import math
from functools import lru_cache
from statistics import NormalDist

import numpy as np

_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _phi(x: float) -> float:
    return 0.0 if math.isinf(x) else math.exp(-0.5 * x * x) * _INV_SQRT_2PI


def _upper_tail(x: float) -> float:
    """P(X > x) for X ~ N(0,1), accurate in the tail."""
    if x == math.inf:
        return 0.0
    if x == -math.inf:
        return 1.0
    return 0.5 * math.erfc(x / _SQRT2)


def _cell_mass(a: float, b: float) -> float:
    """P(a < X < b) without cancellation in either tail."""
    if a >= 0:
        return _upper_tail(a) - _upper_tail(b)
    if b <= 0:
        return _upper_tail(-b) - _upper_tail(-a)
    return 1.0 - _upper_tail(b) - _upper_tail(-a)


def thresholds(levels: np.ndarray) -> np.ndarray:
    """Decision thresholds τ_k = (c_k + c_{k+1}) / 2 of an ascending codebook (float64)."""
    c = np.asarray(levels, dtype=np.float64)
    return 0.5 * (c[:-1] + c[1:])


@lru_cache(maxsize=None)
def _lloyd_max(bits: int) -> tuple[tuple[float, ...], float, int]:
    n_levels = 1 << bits
    nd = NormalDist()
    c = [nd.inv_cdf((k + 0.5) / n_levels) for k in range(n_levels)]
    for it in range(1, 200000):
        t = [-math.inf] + [0.5 * (c[k] + c[k + 1]) for k in range(n_levels - 1)] + [math.inf]
        new = [(_phi(t[k]) - _phi(t[k + 1])) / _cell_mass(t[k], t[k + 1]) for k in range(n_levels)]
        moved = max(abs(a - b) for a, b in zip(c, new))
        c = new
        if moved < 1e-14:
            break
    t = [-math.inf] + [0.5 * (c[k] + c[k + 1]) for k in range(n_levels - 1)] + [math.inf]
    dist = 1.0 - sum(
        (_phi(t[k]) - _phi(t[k + 1])) ** 2 / _cell_mass(t[k], t[k + 1]) for k in range(n_levels)
    )
    return tuple(c), dist, it


def lloyd_max(bits: int) -> np.ndarray:
    """Ascending Lloyd–Max levels for N(0,1) at ``bits`` bits (float64 array of 2^bits)."""
    if not 1 <= bits <= 8:
        raise ValueError("bits must be in 1..8")
    return np.array(_lloyd_max(bits)[0], dtype=np.float64)


def distortion(bits: int) -> float:
    """Mean squared error D_b of the Lloyd–Max quantiser on N(0,1)."""
    return _lloyd_max(bits)[1]


def lloyd_step(levels: np.ndarray) -> np.ndarray:
    """One Lloyd update of an ascending codebook (used to check the fixed point)."""
    c = [float(v) for v in levels]
    n_levels = len(c)
    t = [-math.inf] + [0.5 * (c[k] + c[k + 1]) for k in range(n_levels - 1)] + [math.inf]
    return np.array(
        [(_phi(t[k]) - _phi(t[k + 1])) / _cell_mass(t[k], t[k + 1]) for k in range(n_levels)]
    )


def quantize_distortion(levels: np.ndarray) -> float:
    """E[(X − Q(X))²] of nearest-level quantisation of N(0,1) with the given levels.

    Uses the closed-form cell moments, so it holds for any ascending codebook
    (not only at the Lloyd fixed point).
    """
    c = np.asarray(levels, dtype=np.float64)
    t = [-math.inf] + list(thresholds(c)) + [math.inf]
    total = 0.0
    for k, ck in enumerate(c):
        a, b = t[k], t[k + 1]
        m0 = _cell_mass(a, b)
        m1 = _phi(a) - _phi(b)
        a_phi = 0.0 if math.isinf(a) else a * _phi(a)
        b_phi = 0.0 if math.isinf(b) else b * _phi(b)
        m2 = m0 + a_phi - b_phi
        total += m2 - 2.0 * ck * m1 + ck * ck * m0
    return total
