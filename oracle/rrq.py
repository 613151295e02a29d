"""Random-rotation vector quantisation: encode, decode, rotate, scores (oracle; test infrastructure only).

"Random-rotation quantization" page:

* intro, the scheme, steps 1–3: apply a random orthogonal Π, quantise every
  rotated coordinate independently with one fixed codebook computed once for
  the post-rotation marginal, and at decode time dequantise and apply Πᵀ.
* "History", EDEN bullet: normalise so every coordinate is about N(0,1), then
  the N(0,1) Lloyd–Max codebook; TurboQuant bullet: a constant per-vector scale.
* "Three decoders, one rotation": the MSE decoder maps each (Πx)_i to the
  nearest of 2^b centroids and reconstructs with Πᵀ; the inner-product decoder
  recovers <q, x> from <Πq, code(Πx)> and a normalising scalar.

Readings where the pages are silent:

* per-vector scale is ν = ‖x‖₂ of the input, stored as fp32; the normalised
  coordinate is u = √d·(Πx)_i / ν, which is about N(0,1);
* code_i = #{k : u_i > τ_k} (strict: a value exactly on a threshold takes the
  lower code; u = 0, e.g. for the zero vector, gives code L/2 − 1 for a
  symmetric codebook);
* reconstruction in the rotated domain ŷ_i = (ν/√d)·c[code_i], x̂ = Πᵀ ŷ;
* packed layout: coordinate i occupies bits [i·b, (i+1)·b) of the vector's
  byte string, least significant bit first (b = 4: coordinate 2j in the low
  nibble of byte j);
* attention score s = scale·<q, x̂> = scale·(ν/√d)·Σ_i (Πq)_i·c[code_i]; query
  head h reads KV head ⌊h·Hkv/Hq⌋.

Everything is float64 with the dense rotation matrix; nothing is fused or
reordered.

Pins (tests/test_oracle_pins.py): nearest-centroid brute force for the codes,
a bit-by-bit packer, round-trip NMSE against the Lloyd–Max distortion D_b,
the scores against <q, decode(codes)> computed in the unrotated domain.
"""

from __future__ import annotations

import numpy as np

from .codebook import lloyd_max, thresholds
from .hadamard import rotation_matrix, sylvester
from .rng import bf16_round, rotation_signs


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a float16 / float32 / float64 array."""
    return np.asarray(x).astype(np.float64)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to 'f32' | 'f16' | 'bf16' (nearest even), returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "f16":
        return x.astype(np.float16).astype(np.float64)
    if dtype == "bf16":
        return bf16_round(x)
    raise ValueError(dtype)


def default_levels(bits: int) -> np.ndarray:
    return lloyd_max(bits)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """[N, d] integer codes -> [N, d*bits/8] uint8, coordinate i at bits [i*b, (i+1)*b), LSB first."""
    codes = np.asarray(codes, dtype=np.int64)
    n, d = codes.shape
    if (d * bits) % 8:
        raise ValueError("d*bits must be a multiple of 8")
    bitplanes = ((codes[:, :, None] >> np.arange(bits)[None, None, :]) & 1).astype(np.uint8)
    return np.packbits(bitplanes.reshape(n, d * bits), axis=1, bitorder="little")


def unpack_codes(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of pack_codes: [N, d*bits/8] uint8 -> [N, d] int64."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    flat = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * bits].reshape(n, d, bits)
    return (flat.astype(np.int64) << np.arange(bits)[None, None, :]).sum(axis=2)


def rotate(x, seed: int, inverse: bool = False) -> np.ndarray:
    """Πx (or Πᵀx) of every row, float64."""
    x = as_f64(x)
    p = rotation_matrix(seed, x.shape[-1])
    return x @ (p if inverse else p.T)


class Encoded:
    """Oracle encode result.

    codes  [N, d] int64   — unpacked codes
    packed [N, d*b/8] u8  — packed codes
    norms  [N] float32    — stored per-vector scale fp32(‖x‖₂)
    norm64 [N] float64    — ‖x‖₂ before rounding
    y      [N, d] float64 — rotated vectors Πx
    u      [N, d] float64 — normalised rotated coordinates √d·Πx/‖x‖
    """

    def __init__(self, codes, packed, norms, norm64, y, u):
        self.codes, self.packed, self.norms, self.norm64, self.y, self.u = (
            codes, packed, norms, norm64, y, u)


def encode(x, bits: int, seed: int, levels=None) -> Encoded:
    """Encode rows of x ([N, d]) at ``bits`` bits with rotation seed ``seed``.

    ``levels``: ascending codebook (float64 or float32 values); default is the
    N(0,1) Lloyd–Max codebook.
    """
    x = as_f64(x)
    n, d = x.shape
    c = default_levels(bits) if levels is None else np.asarray(levels, dtype=np.float64)
    tau = thresholds(c)
    # √d·Πx = H·(D·x) exactly (Π = H·D/√d); with the ±1 matrix H the fp64
    # products are exact and the sums of fp16/bf16 inputs are exact too, so a
    # coordinate that lies exactly on a threshold (e.g. u = 0) is decided by the
    # tie rule above rather than by rounding noise.
    hd = sylvester(d) * rotation_signs(seed, d)[None, :]
    y_sqrt_d = x @ hd.T
    y = y_sqrt_d / np.sqrt(d)
    nu = np.sqrt(np.sum(x * x, axis=1))
    u = np.zeros_like(y)
    nzr = nu > 0
    u[nzr] = y_sqrt_d[nzr] / nu[nzr, None]
    # code = number of thresholds strictly below u
    codes = np.searchsorted(tau, u.ravel(), side="left").reshape(n, d).astype(np.int64)
    return Encoded(codes, pack_codes(codes, bits), nu.astype(np.float32), nu, y, u)


def dequantize_rotated(codes: np.ndarray, norms, bits: int, levels=None) -> np.ndarray:
    """ŷ = (ν/√d)·c[code] in the rotated domain, float64 [N, d]."""
    codes = np.asarray(codes, dtype=np.int64)
    d = codes.shape[1]
    c = default_levels(bits) if levels is None else np.asarray(levels, dtype=np.float64)
    nu = as_f64(norms)
    return (nu[:, None] / np.sqrt(d)) * c[codes]


def decode_exact(packed, norms, bits: int, d: int, seed: int, levels=None) -> np.ndarray:
    """x̂ = Πᵀ ŷ in float64 (before rounding to the output dtype)."""
    codes = unpack_codes(packed, bits, d)
    yhat = dequantize_rotated(codes, norms, bits, levels)
    return rotate(yhat, seed, inverse=True)


def decode(packed, norms, bits: int, d: int, seed: int, levels=None, out_dtype: str = "f16") -> np.ndarray:
    """Reconstruction rounded to ``out_dtype`` (returned as float64 values)."""
    return round_to(decode_exact(packed, norms, bits, d, seed, levels), out_dtype)


def kv_group(h: int, hq: int, hkv: int) -> int:
    """KV head read by query head h: ⌊h·Hkv/Hq⌋ (consecutive groups)."""
    return (h * hkv) // hq


def scores(q, packed, norms, t_len: int, hkv: int, d: int, bits: int, seed: int,
           levels=None, scale: float = 1.0) -> np.ndarray:
    """Attention scores s[h, t] = scale·(ν_{t,g}/√d)·Σ_i (Πq_h)_i·c[code_{t,g,i}], float64 [Hq, T].

    q: [Hq, d] (unrotated); packed: [T*Hkv, d*b/8] with row n = t*Hkv + g;
    norms: [T*Hkv].
    """
    q = as_f64(q)
    hq = q.shape[0]
    c = default_levels(bits) if levels is None else np.asarray(levels, dtype=np.float64)
    qr = rotate(q, seed)  # Πq
    codes = unpack_codes(packed, bits, d).reshape(t_len, hkv, d)
    nu = as_f64(norms).reshape(t_len, hkv)
    levels_of = c[codes]  # [T, Hkv, d]
    out = np.empty((hq, t_len), dtype=np.float64)
    for h in range(hq):
        g = kv_group(h, hq, hkv)
        out[h] = scale * (nu[:, g] / np.sqrt(d)) * (levels_of[:, g, :] @ qr[h])
    return out


def score_tolerance_scale(q, packed, norms, t_len: int, hkv: int, d: int, bits: int,
                          levels=None) -> np.ndarray:
    """‖q_h‖·‖k̂_{t,g(h)}‖ for every (h, t): the Cauchy–Schwarz scale of a score."""
    q = as_f64(q)
    hq = q.shape[0]
    c = default_levels(bits) if levels is None else np.asarray(levels, dtype=np.float64)
    codes = unpack_codes(packed, bits, d).reshape(t_len, hkv, d)
    nu = as_f64(norms).reshape(t_len, hkv)
    khat_norm = (nu / np.sqrt(d)) * np.sqrt(np.sum(c[codes] ** 2, axis=2))
    qn = np.sqrt(np.sum(q * q, axis=1))
    return np.stack([qn[h] * khat_norm[:, kv_group(h, hq, hkv)] for h in range(hq)])
