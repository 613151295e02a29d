"""Sphere marginal and DRIVE scales (oracle; test infrastructure only).

Used only to pin the rotation against what the "Random-rotation quantization"
page states; not part of the GPU path.

* "Why rotation works": a uniformly random rotation sends x to a uniform point
  on the sphere of radius ‖x‖; each coordinate of a unit-sphere point has mean
  0, standard deviation 1/√d and marginal density
      f(x) = Γ(d/2) / (√π · Γ((d−1)/2)) · (1 − x²)^((d−3)/2),   −1 < x < 1,
  which tends to N(0, 1/d) (at d = 1000 the standard deviation is ≈ 0.032).
  (The extracted text lost the LaTeX thin spaces; the reading above restores
  them.)
* "History", DRIVE bullet: one bit per coordinate, sign(R(x)), plus a scale;
  S = ‖R(x)‖₁/d is biased and MSE-optimal, S = ‖x‖₂²/‖R(x)‖₁ is unbiased.
  "Three decoders, one rotation", mean decoder: x̂ = S·Πᵀ·sign(Πx).
"""

from __future__ import annotations

import math

import numpy as np

from .rrq import as_f64, pack_codes, rotate


def marginal_density(x, d: int) -> np.ndarray:
    """Density of one coordinate of a uniform point on the unit sphere in R^d (d >= 3)."""
    x = np.asarray(x, dtype=np.float64)
    log_norm = math.lgamma(d / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((d - 1) / 2.0)
    out = np.zeros_like(x)
    inside = np.abs(x) < 1.0
    out[inside] = np.exp(log_norm + 0.5 * (d - 3) * np.log1p(-x[inside] ** 2))
    return out


def drive_scale_biased(rx) -> np.ndarray:
    """S = ‖R(x)‖₁ / d for each row of the rotated vectors R(x)."""
    rx = as_f64(rx)
    return np.sum(np.abs(rx), axis=-1) / rx.shape[-1]


def drive_scale_unbiased(x, rx) -> np.ndarray:
    """S = ‖x‖₂² / ‖R(x)‖₁ for each row."""
    x, rx = as_f64(x), as_f64(rx)
    return np.sum(x * x, axis=-1) / np.sum(np.abs(rx), axis=-1)


def drive_mean_decode(rotation: np.ndarray, bits, scale) -> np.ndarray:
    """x̂ = S·Πᵀ·(2·bit − 1) for rows of sign bits ("Three decoders, one
    rotation", mean decoder)."""
    p = as_f64(rotation)
    sgn = 2.0 * np.asarray(bits, dtype=np.float64) - 1.0
    return np.asarray(scale, dtype=np.float64)[..., None] * (sgn @ p)


def drive_decode(rotation: np.ndarray, x, scale) -> np.ndarray:
    """x̂ = S·Πᵀ·sign(Πx) for rows of x.  sign(0) is taken as −1: the page
    leaves it open, and −1 is the b-bit encoder's rule with τ = 0 (a value on
    a threshold takes the lower code)."""
    x = as_f64(x)
    p = as_f64(rotation)
    return drive_mean_decode(p, (x @ p.T) > 0, scale)


class DriveEncoded:
    """signs [N, d] int64 (1 where (Πx)_i > 0), packed [N, d/8] u8 (LSB first),
    scale [N] float64 (S), stored [N] float32 (fp32(S·√d), the per-vector value
    that the rrq 1-bit decoder and score path read as their norm)."""

    def __init__(self, signs, packed, scale, stored, rx):
        self.signs, self.packed, self.scale, self.stored, self.rx = signs, packed, scale, stored, rx


def drive_encode(x, seed: int, unbiased: bool) -> DriveEncoded:
    """DRIVE's one-bit encoder ("History", DRIVE bullet): sign(Πx) and the scale S.

    S = ‖Πx‖₁/d (biased, MSE-optimal) or S = ‖x‖₂²/‖Πx‖₁ (unbiased).  A code is
    1 when (Πx)_i > 0 (strict, the rule of the b-bit encoder with τ = 0), so
    with the codebook {−1, +1} and the stored value S·√d the b-bit decoder
    returns S·Πᵀ·sign(Πx), the mean decoder of "Three decoders, one rotation".
    """
    x = as_f64(x)
    d = x.shape[-1]
    rx = rotate(x, seed)
    with np.errstate(invalid="ignore", divide="ignore"):  # x = 0: S = 0 below
        s = drive_scale_unbiased(x, rx) if unbiased else drive_scale_biased(rx)
    s = np.where(np.sum(np.abs(rx), axis=-1) > 0, s, 0.0)
    signs = (rx > 0).astype(np.int64)
    stored = (s * math.sqrt(d)).astype(np.float32)
    return DriveEncoded(signs, pack_codes(signs, 1), s, stored, rx)
