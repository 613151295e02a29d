"""QJL 1-bit sign sketch of the quantisation residual (oracle; test infrastructure only).

"Random-rotation quantization" page:

* "History", QJL bullet: a DRIVE-style one-bit construction for attention keys,
  made unbiased through residuals; TurboQuant bullet: a residual chain — a
  biased (b−1)-bit MSE quantiser followed by an unbiased 1-bit one.
* "Three decoders, one rotation", inner-product decoder: <q, x> is recovered
  from <Πq, sign(·)> with a normalising scalar.
* "Bias vs unbiasedness": MSE-optimal quantisers shrink, so their inner
  products are biased low; the residual chain removes the bias.

Readings (the pages give no formulas for this stage):

* residual in the rotated domain: r = Πx − ŷ with ŷ the MSE reconstruction the
  decoder would produce from the stored fp32 norm;
* projection: v = S·r with S a d×d matrix of bf16-rounded standard normals
  (``rng.qjl_gaussian``); stored bit_i = [v_i > 0] (LSB first, d bits per
  vector) and ρ = fp32(‖r‖₂);
* estimator: <q', r> ≈ √(π/2)/m · ρ · Σ_i (S q')_i · (2·bit_i − 1), m = d rows,
  q' = Πq.  The constant follows from E|g| = √(2/π) for g ~ N(0,1) — the
  same quantity as the 1-bit Lloyd–Max level in the EDEN bullet.

Pins (tests/test_oracle_pins.py): unbiasedness of the estimator by Monte Carlo
over independent Gaussian S; S·r computed as an explicit double loop on tiny
inputs.
"""

from __future__ import annotations

import numpy as np

from . import rrq
from .rrq import as_f64


class QJLEncoded:
    """enc: the MSE Encoded; r [N, d] float64; v [N, d] float64; bits [N, d/8] u8; rnorm [N] float32."""

    def __init__(self, enc, r, v, bits, rnorm):
        self.enc, self.r, self.v, self.bits, self.rnorm = enc, r, v, bits, rnorm


def residual(x, bits: int, seed: int, levels=None):
    enc = rrq.encode(x, bits, seed, levels)
    yhat = rrq.dequantize_rotated(enc.codes, enc.norms, bits, levels)
    return enc, enc.y - yhat


def encode(x, bits: int, seed: int, s_matrix: np.ndarray, levels=None) -> QJLEncoded:
    enc, r = residual(x, bits, seed, levels)
    s = as_f64(s_matrix)
    v = r @ s.T  # v_i = sum_j S[i, j] r_j
    sign_bits = (v > 0).astype(np.uint8)
    packed = np.packbits(sign_bits, axis=1, bitorder="little")
    rho = np.sqrt(np.sum(r * r, axis=1))
    return QJLEncoded(enc, r, v, packed, rho.astype(np.float32))


def unpack_signs(packed: np.ndarray, d: int) -> np.ndarray:
    """[N, d/8] uint8 -> [N, d] float64 of +-1."""
    b = np.unpackbits(np.asarray(packed, dtype=np.uint8), axis=1, bitorder="little")[:, :d]
    return 2.0 * b.astype(np.float64) - 1.0


def estimate_residual_dot(q_rot, s_matrix, packed_signs, rnorm) -> np.ndarray:
    """√(π/2)/m · ρ_n · <S q', sign_n> for every stored vector n; q_rot = Πq (length d)."""
    s = as_f64(s_matrix)
    m, d = s.shape
    sq = s @ as_f64(q_rot)
    signs = unpack_signs(packed_signs, d)
    return np.sqrt(np.pi / 2.0) / m * as_f64(rnorm) * (signs @ sq)


def scores_unbiased(q, packed, norms, qjl_bits, rnorm, t_len: int, hkv: int, d: int, bits: int,
                    seed: int, s_matrix, levels=None, scale: float = 1.0) -> np.ndarray:
    """Unbiased attention scores on TurboQuant-style keys, float64 [Hq, T].

    "Random-rotation quantization" page, TurboQuant bullet (an MSE quantiser
    followed by an unbiased one-bit stage on the residual) and "Three decoders,
    one rotation", inner-product decoder:
        s[h, t] = scale · ( <q_h, x̂_{t,g}> + √(π/2)/m · ρ_{t,g} · <S Π q_h, sign_{t,g}> ),
    g = ⌊h·Hkv/Hq⌋, the first term the b-bit MSE score (``rrq.scores``), the
    second the residual estimate (``estimate_residual_dot``).  Rows of packed /
    norms / qjl_bits / rnorm are n = t·Hkv + g.
    """
    q = as_f64(q)
    hq = q.shape[0]
    out = rrq.scores(q, packed, norms, t_len, hkv, d, bits, seed, levels, scale)
    qr = rrq.rotate(q, seed)
    qb = np.asarray(qjl_bits, dtype=np.uint8).reshape(t_len, hkv, d // 8)
    rn = as_f64(rnorm).reshape(t_len, hkv)
    for h in range(hq):
        g = rrq.kv_group(h, hq, hkv)
        out[h] += scale * estimate_residual_dot(qr[h], s_matrix, qb[:, g, :], rn[:, g])
    return out
