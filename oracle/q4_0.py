"""Rotate-then-q4_0 ("Attn-rot", TurboQuant lite) encode and decode (oracle; test infrastructure only).

"Attn-rot (TurboQuant lite) in llama.cpp" page, section "What kind of beast is
Attn-rot": rotate the K and V vectors first, then quantise the cache with an
ordinary block format; section "How to use it", the note on batch-quantisable
types: q4_0 first of all (also q4_1, q5_0, q5_1).  The rotation is the same
randomized Hadamard transform as the main scheme ("Random-rotation
quantization" page, "Why rotation works").

The page names q4_0 but does not define it.  The reading used (the public
llama.cpp/GGML q4_0 block, kept identical for interoperability):

* blocks of 32 consecutive (rotated) coordinates;
* the decisions are taken in fp32, the precision of the format's reference
  arithmetic (the pages fix none): y is rounded to fp32 first;
* m = the block element of largest magnitude, with its sign (first index on
  ties; +0 when every element is ±0, as the public reference quantiser starts
  from +0); Δ = m / −8 (exact); inv = fp32(1/Δ) (0 when Δ = 0);
* q_j = min(15, ⌊fp32(fp32(y_j·inv) + 8.5)⌋) (the argument is ≥ 0.5 since
  |y_j·inv| ≤ 8);
* stored: fp16(Δ) (2 bytes, little endian) then 16 bytes; byte j holds q_j in
  its low nibble and q_{j+16} in its high nibble — 18 bytes per block;
* decode: (q_j − 8)·fp16(Δ), then Πᵀ when the vector was rotated.

The rotation here is orthonormal: y = Πx = H·D·x/√d.

Pins (tests/test_oracle_pins.py): hand-worked blocks (all equal, a single
outlier, all zero, exactly representable grids), rotate=0 round trip exact on
grid inputs, rotate=1 equivalence with rotate=0 applied to Πx.
"""

from __future__ import annotations

import numpy as np

from .rrq import as_f64, round_to, rotate

BLOCK = 32
BLOCK_BYTES = 18


class Q4Encoded:
    """blocks [N, d/32*18] uint8; delta [N, d/32] float32 (before fp16); q [N, d] int64; y [N, d] float64."""

    def __init__(self, blocks, delta, q, y, ratio):
        self.blocks, self.delta, self.q, self.y, self.ratio = blocks, delta, q, y, ratio


def encode(x, seed: int, rotate_first: bool = True) -> Q4Encoded:
    x = as_f64(x)
    n, d = x.shape
    if d % BLOCK:
        raise ValueError("d must be a multiple of 32")
    y = rotate(x, seed) if rotate_first else x.copy()
    nb = d // BLOCK
    yb = y.reshape(n, nb, BLOCK)
    y32 = yb.astype(np.float32)
    idx = np.argmax(np.abs(y32), axis=2)  # first index on ties
    m = np.take_along_axis(y32, idx[:, :, None], axis=2)[:, :, 0]
    m = np.where(np.abs(m) > 0, m, np.float32(0.0)).astype(np.float32)  # all-zero block: +0
    delta = (m / np.float32(-8.0)).astype(np.float32)
    inv = np.zeros_like(delta)
    nz = delta != 0
    inv[nz] = np.float32(1.0) / delta[nz]
    r32 = (y32 * inv[:, :, None]).astype(np.float32) + np.float32(8.5)
    q = np.minimum(15, np.maximum(0, np.floor(r32))).astype(np.int64)
    # the same quantity in fp64, for measuring distances to code boundaries
    ratio = yb * inv[:, :, None].astype(np.float64) + 8.5
    # serialise: fp16 delta, then nibbles (j low, j+16 high)
    blocks = np.zeros((n, nb, BLOCK_BYTES), dtype=np.uint8)
    dh = delta.astype(np.float16).view(np.uint16)
    blocks[:, :, 0] = (dh & 0xFF).astype(np.uint8)
    blocks[:, :, 1] = (dh >> 8).astype(np.uint8)
    blocks[:, :, 2:] = (q[:, :, :16] | (q[:, :, 16:] << 4)).astype(np.uint8)
    return Q4Encoded(blocks.reshape(n, nb * BLOCK_BYTES), delta, q.reshape(n, d), y, ratio.reshape(n, d))


def parse_blocks(blocks: np.ndarray, d: int):
    """-> (fp16 deltas as float64 [N, d/32], codes [N, d] int64)."""
    b = np.asarray(blocks, dtype=np.uint8)
    n = b.shape[0]
    nb = d // BLOCK
    b = b.reshape(n, nb, BLOCK_BYTES)
    dh = (b[:, :, 0].astype(np.uint16) | (b[:, :, 1].astype(np.uint16) << 8)).view(np.float16)
    lo = (b[:, :, 2:] & 0x0F).astype(np.int64)
    hi = (b[:, :, 2:] >> 4).astype(np.int64)
    q = np.concatenate([lo, hi], axis=2).reshape(n, d)
    return dh.astype(np.float64), q


def decode_exact(blocks, d: int, seed: int, rotate_first: bool = True) -> np.ndarray:
    dh, q = parse_blocks(blocks, d)
    n = q.shape[0]
    yhat = ((q.reshape(n, d // BLOCK, BLOCK) - 8) * dh[:, :, None]).reshape(n, d)
    return rotate(yhat, seed, inverse=True) if rotate_first else yhat


def decode(blocks, d: int, seed: int, rotate_first: bool = True, out_dtype: str = "f16") -> np.ndarray:
    return round_to(decode_exact(blocks, d, seed, rotate_first), out_dtype)
