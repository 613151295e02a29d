"""Counter-based random numbers the method draws (oracle side; test infrastructure only).

The pages fix no generator: the "Random-rotation quantization" page, section
"Why rotation works", only says the rotation in practice is a *randomized*
Hadamard transform.  The reading used here (and independently on the GPU side)
is:

* SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; constants as in Vigna's public reference
  implementation).  Output number ``c`` (c = 0, 1, ...) of a generator seeded
  with ``seed`` is ``mix(seed + (c + 1) * GAMMA)``.
* Rotation sign s_i (i = 0..d-1) is -1 when bit 63 of output ``i`` is set,
  else +1.  One sign vector per call, shared by every vector of that call
  ("Three decoders, one rotation": the rotation is the shared encoder).
* QJL matrix entry S[i, j] (row-major element e = i*d + j) is a standard normal
  by Box–Muller from outputs 2e and 2e+1, rounded to bf16 (nearest even).

Pins: ``splitmix64`` is pinned to the published first outputs for seed 1234567
(tests/golden/splitmix64_vectors.txt).  The sign and Gaussian constructions on
top of it are this library's own definition ("parity unpinned" against the pages,
which name no generator); the Gaussian is pinned statistically (moments).
"""

from __future__ import annotations

import math

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15  # SplitMix64 increment (golden-ratio constant)


def _mix(z: int) -> int:
    """SplitMix64 output finalizer on a 64-bit state value."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64(seed: int, count: int, start: int = 0) -> list[int]:
    """Outputs ``start .. start+count-1`` of SplitMix64 seeded with ``seed``."""
    seed &= MASK64
    return [_mix(seed + (c + 1) * GAMMA) for c in range(start, start + count)]


def rotation_signs(seed: int, d: int) -> np.ndarray:
    """Diagonal of D (float64 array of +-1): s_i = -1 iff bit 63 of output i is set."""
    out = splitmix64(seed, d)
    return np.array([-1.0 if (w >> 63) & 1 else 1.0 for w in out], dtype=np.float64)


def bf16_round(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (ties to even), returned as float64.

    Done directly from float64 (no float32 intermediate, so no double rounding):
    bf16 keeps 8 significant bits and float32's exponent range.
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = (v != 0) & np.isfinite(v)
    m, e = np.frexp(v[nz])  # v = m * 2**e, 0.5 <= |m| < 1
    # normal bf16: 8 significant bits -> quantum 2**(e-8); below 2**-126 the
    # quantum is fixed at 2**-133 (subnormals)
    q_exp = np.maximum(e - 8, -133)
    r = np.rint(np.ldexp(v[nz], -q_exp))  # rint is round-half-even
    out[nz] = np.ldexp(r, q_exp)
    out[~np.isfinite(v)] = v[~np.isfinite(v)]
    big = np.abs(out) > 3.3895313892515355e38  # above max finite bf16
    out[big] = np.copysign(np.inf, out[big])
    return out


def bf16_bits(v: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of float64 values that are already bf16-exact."""
    f32 = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def qjl_gaussian(seed: int, d: int) -> np.ndarray:
    """The d x d QJL projection S (float64 array holding bf16-exact values).

    Entry e = i*d + j: u1, u2 = the top 53 bits of outputs 2e and 2e+1 as
    uniforms in [0, 1); z = sqrt(-2 ln(1 - u1)) * cos(2 pi u2) (Box–Muller,
    1 - u1 in (0, 1] so the log is finite); S[i, j] = bf16(z).
    """
    n = d * d
    words = splitmix64(seed, 2 * n)
    z = np.empty(n, dtype=np.float64)
    two_pi = 2.0 * math.pi
    for e in range(n):
        u1 = (words[2 * e] >> 11) * (1.0 / 9007199254740992.0)
        u2 = (words[2 * e + 1] >> 11) * (1.0 / 9007199254740992.0)
        z[e] = math.sqrt(-2.0 * math.log(1.0 - u1)) * math.cos(two_pi * u2)
    return bf16_round(z).reshape(d, d)
