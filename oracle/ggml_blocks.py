"""Rotate-then-block-quantise with the other GGML block types: q4_1, q5_0, q5_1, q8_0
(oracle; test infrastructure only).

"Attn-rot (TurboQuant lite) in llama.cpp" page, section "How to use it": besides
q4_0, the batch-quantisable cache types q4_1, q5_0 and q5_1 (and q8_0, the
8-bit type the same page lists among the cache types).  The rotation is the
randomized Hadamard transform of the main scheme ("Random-rotation
quantization" page, "Why rotation works"), orthonormal here: y = Πx.

The page names these types without defining them.  The reading used is the
public llama.cpp/GGML block of each, kept identical for interoperability, with
the decisions taken in fp32 (y rounded to fp32 first; every product, sum and
quotient below rounded to fp32, no fused multiply-add), in blocks of 32
consecutive coordinates:

* q4_1 (20 bytes): lo = min y, hi = max y (the first such element in index
  order, so that of −0 and +0 the first is kept); Δ = (hi − lo)/15; inv = 1/Δ (0 when
  Δ = 0); q_j = min(15, ⌊(y_j − lo)·inv + 0.5⌋); stored fp16(Δ), fp16(lo), then
  byte j = q_j | q_{j+16} << 4.  Decode: q_j·Δ + lo.
* q5_0 (22 bytes): m = the element of largest |y| with its sign (first on ties;
  +0 when the block is all zeros);
  Δ = m/−16; q_j = min(31, ⌊y_j·inv + 16.5⌋); stored fp16(Δ), then a 32-bit
  little-endian word whose bit j is bit 4 of q_j (j = 0..31), then byte
  j = (q_j & 15) | (q_{j+16} & 15) << 4.  Decode: (q_j − 16)·Δ.
* q5_1 (24 bytes): as q4_1 with Δ = (hi − lo)/31 and q_j = ⌊(y_j − lo)·inv + 0.5⌋
  (at most 31); stored fp16(Δ), fp16(lo), the high-bit word, then the nibbles.
  Decode: q_j·Δ + lo.
* q8_0 (34 bytes): a = max |y|; Δ = a/127; q_j = round(y_j·inv), halves away
  from zero, as a signed byte; stored fp16(Δ) then the 32 bytes.  Decode: q_j·Δ.

Decoding uses the stored fp16 values; the oracle decodes in float64.

Pins (tests/test_oracle_pins.py): hand-worked blocks for every type
(tests/golden/ggml_blocks.txt), exact round trips of grid inputs, the
rotate = 1 encoding equal to the rotate = 0 encoding of Πx, and q5_1/q8_0 errors
below their half-step bounds.
"""

from __future__ import annotations

import numpy as np

from .rrq import as_f64, round_to, rotate

BLOCK = 32
FORMATS = ("q4_1", "q5_0", "q5_1", "q8_0")
BLOCK_BYTES = {"q4_1": 20, "q5_0": 22, "q5_1": 24, "q8_0": 34}
F32 = np.float32


class BlockEncoded:
    """blocks [N, d/32·bytes] uint8; q [N, d] int64 codes; y [N, d] float64 (the
    rotated values); scale32 / min32 [N, d/32] float32 (before fp16 rounding;
    min32 is 0 for the formats without one); margin [N, d] float64: distance of
    the exact decision quantity to its nearest rounding boundary, in code units
    (for judging codes decided differently by a few fp32 ulps)."""

    def __init__(self, fmt, blocks, q, y, scale32, min32, margin):
        self.fmt, self.blocks, self.q, self.y = fmt, blocks, q, y
        self.scale32, self.min32, self.margin = scale32, min32, margin


def _signed_absmax(y32: np.ndarray) -> np.ndarray:
    """The element of largest |y| with its sign, first index on ties, over the last
    axis; +0 for a block of zeros (whatever the signs of its zeros)."""
    idx = np.argmax(np.abs(y32), axis=-1)
    m = np.take_along_axis(y32, idx[..., None], axis=-1)[..., 0]
    return np.where(np.abs(m) > 0, m, F32(0.0)).astype(F32)


def _first_extreme(y32: np.ndarray, largest: bool) -> np.ndarray:
    """The first element (in index order) of smallest or largest value: −0 and +0
    compare equal, so the first of them is kept."""
    idx = np.argmax(y32, axis=-1) if largest else np.argmin(y32, axis=-1)
    return np.take_along_axis(y32, idx[..., None], axis=-1)[..., 0]


def _inverse(delta: np.ndarray) -> np.ndarray:
    inv = np.zeros_like(delta)
    nz = delta != 0
    inv[nz] = F32(1.0) / delta[nz]
    return inv


def block_decisions(y32: np.ndarray, fmt: str, pick=None):
    """Codes of fp32 blocks y32 [..., 32] under `fmt`, with the fp32 scalars.

    -> (q int64 [..., 32], scale32, min32, margin).  `pick` (optional, absmax
    formats only): the index of the element to take the scale from, instead of
    the first of largest magnitude.
    """
    y32 = np.asarray(y32, dtype=F32)
    y64 = y32.astype(np.float64)
    zero = np.zeros(y32.shape[:-1], dtype=F32)
    if fmt in ("q4_1", "q5_1"):
        levels = 15 if fmt == "q4_1" else 31
        lo = _first_extreme(y32, largest=False)
        hi = _first_extreme(y32, largest=True)
        delta = ((hi - lo).astype(F32) / F32(levels)).astype(F32)
        inv = _inverse(delta)
        t = ((y32 - lo[..., None]).astype(F32) * inv[..., None]).astype(F32)
        r = (t + F32(0.5)).astype(F32)
        q = np.minimum(levels, np.floor(r)).astype(np.int64)
        exact = (y64 - lo[..., None].astype(np.float64)) * inv[..., None].astype(np.float64) + 0.5
        margin = np.abs(exact - np.round(exact))
        return q, delta, lo, margin
    if fmt == "q5_0":
        m = (_signed_absmax(y32) if pick is None
             else np.take_along_axis(y32, np.asarray(pick)[..., None], axis=-1)[..., 0])
        delta = (m / F32(-16.0)).astype(F32)
        inv = _inverse(delta)
        r = ((y32 * inv[..., None]).astype(F32) + F32(16.5)).astype(F32)
        q = np.minimum(31, np.floor(r)).astype(np.int64)
        exact = y64 * inv[..., None].astype(np.float64) + 16.5
        margin = np.abs(exact - np.round(exact))
        return q, delta, zero, margin
    if fmt == "q8_0":
        a = np.max(np.abs(y32), axis=-1)
        delta = (a / F32(127.0)).astype(F32)
        inv = _inverse(delta)
        t = (y32 * inv[..., None]).astype(F32)
        q = (np.sign(t) * np.floor(np.abs(t).astype(np.float64) + 0.5)).astype(np.int64)
        exact = y64 * inv[..., None].astype(np.float64)
        margin = np.abs(np.abs(exact) - np.floor(np.abs(exact)) - 0.5)
        return q, delta, zero, margin
    raise ValueError(f"unknown block type {fmt!r}")


def _fp16_bytes(v: np.ndarray) -> np.ndarray:
    h = np.asarray(v, dtype=F32).astype(np.float16).view(np.uint16)
    return np.stack([(h & 0xFF).astype(np.uint8), (h >> 8).astype(np.uint8)], axis=-1)


def serialize(fmt: str, q: np.ndarray, scale32: np.ndarray, min32: np.ndarray) -> np.ndarray:
    """Block bytes [..., BLOCK_BYTES[fmt]] from codes [..., 32] and fp32 scalars."""
    parts = [_fp16_bytes(scale32)]
    if fmt in ("q4_1", "q5_1"):
        parts.append(_fp16_bytes(min32))
    if fmt in ("q5_0", "q5_1"):
        high = ((q >> 4) & 1).astype(np.uint64)
        word = np.sum(high << np.arange(BLOCK, dtype=np.uint64), axis=-1)
        parts.append(np.stack([((word >> np.uint64(8 * k)) & np.uint64(0xFF)).astype(np.uint8)
                               for k in range(4)], axis=-1))
    if fmt == "q8_0":
        parts.append((q & 0xFF).astype(np.uint8))
    else:
        lo4 = q[..., :16] & 15
        hi4 = q[..., 16:] & 15
        parts.append((lo4 | (hi4 << 4)).astype(np.uint8))
    return np.concatenate(parts, axis=-1)


def encode(x, seed: int, fmt: str, rotate_first: bool = True) -> BlockEncoded:
    x = as_f64(x)
    n, d = x.shape
    if d % BLOCK:
        raise ValueError("d must be a multiple of 32")
    y = rotate(x, seed) if rotate_first else x.copy()
    nb = d // BLOCK
    y32 = y.reshape(n, nb, BLOCK).astype(F32)
    q, s32, m32, margin = block_decisions(y32, fmt)
    blocks = serialize(fmt, q, s32, m32)
    return BlockEncoded(fmt, blocks.reshape(n, nb * BLOCK_BYTES[fmt]), q.reshape(n, d), y,
                        s32, m32, margin.reshape(n, d))


def parse_blocks(blocks: np.ndarray, d: int, fmt: str):
    """-> (fp16 scale, fp16 min (0 when absent), codes [N, d] int64), scalars [N, d/32] float64."""
    nbytes = BLOCK_BYTES[fmt]
    b = np.asarray(blocks, dtype=np.uint8)
    n = b.shape[0]
    nb = d // BLOCK
    b = b.reshape(n, nb, nbytes)

    def f16(k):
        return (b[:, :, k].astype(np.uint16) | (b[:, :, k + 1].astype(np.uint16) << 8)).view(
            np.float16).astype(np.float64)

    scale = f16(0)
    off = 2
    mn = np.zeros_like(scale)
    if fmt in ("q4_1", "q5_1"):
        mn = f16(2)
        off = 4
    high = np.zeros((n, nb, BLOCK), dtype=np.int64)
    if fmt in ("q5_0", "q5_1"):
        word = np.zeros((n, nb), dtype=np.uint64)
        for k in range(4):
            word |= b[:, :, off + k].astype(np.uint64) << np.uint64(8 * k)
        high = ((word[:, :, None] >> np.arange(BLOCK, dtype=np.uint64)) & np.uint64(1)).astype(np.int64)
        off += 4
    if fmt == "q8_0":
        q = b[:, :, off:off + BLOCK].view(np.int8).astype(np.int64)
    else:
        qs = b[:, :, off:off + 16]
        q = np.concatenate([qs & 15, qs >> 4], axis=2).astype(np.int64) | (high << 4)
    return scale, mn, q.reshape(n, d)


def dequantize(blocks, d: int, fmt: str) -> np.ndarray:
    """Block values in the (rotated) domain, float64 [N, d]."""
    scale, mn, q = parse_blocks(blocks, d, fmt)
    n = q.shape[0]
    qb = q.reshape(n, d // BLOCK, BLOCK).astype(np.float64)
    if fmt in ("q4_1", "q5_1"):
        v = qb * scale[:, :, None] + mn[:, :, None]
    elif fmt == "q5_0":
        v = (qb - 16.0) * scale[:, :, None]
    else:
        v = qb * scale[:, :, None]
    return v.reshape(n, d)


def decode_exact(blocks, d: int, seed: int, fmt: str, rotate_first: bool = True) -> np.ndarray:
    yhat = dequantize(blocks, d, fmt)
    return rotate(yhat, seed, inverse=True) if rotate_first else yhat


def decode(blocks, d: int, seed: int, fmt: str, rotate_first: bool = True,
           out_dtype: str = "f16") -> np.ndarray:
    return round_to(decode_exact(blocks, d, seed, fmt, rotate_first), out_dtype)
