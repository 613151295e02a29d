"""Decode-time attention over a fully quantised K/V cache (oracle; test infrastructure only).

"Attn-rot (TurboQuant lite) in llama.cpp" page, section "What kind of beast is
Attn-rot": both the keys (K) and the values (V) of the attention are
quantised after a rotation.  "Random-rotation quantization" page, "Three
decoders, one rotation": the MSE decoder (nearest Lloyd–Max centroid per
rotated coordinate, x̃ = Πᵀ(…)) is the one for KV-cache compression.

For one decode step with query heads q_h and a cache of T tokens × Hkv heads:
    s[h, t] = scale · <q_h, k̂_{t,g}>             (the b-bit score, ``rrq.scores``),
    p[h, t] = exp(s[h, t] − max_t s[h, ·]) / Σ_t exp(s[h, t] − max_t s[h, ·]),
    out[h]  = Σ_t p[h, t] · v̂_{t,g},   g = ⌊h·Hkv/Hq⌋,
with k̂, v̂ the MSE reconstructions (``rrq.decode_exact``) under their own
rotation seeds and codebooks.  Everything in float64.

Pins (tests/test_oracle_pins.py): one token gives that token's v̂; a zero query
gives the mean of v̂; a large scale concentrates the weight on the top-scoring
token; permuting the tokens changes nothing.
"""

from __future__ import annotations

import numpy as np

from . import rrq
from .rrq import as_f64


def decode_attention(q, k_packed, k_norms, v_packed, v_norms, t_len: int, hkv: int, d: int,
                     k_bits: int, v_bits: int, k_seed: int, v_seed: int, k_levels=None,
                     v_levels=None, scale: float = 1.0, return_weights: bool = False):
    """out [Hq, d] float64.  Cache rows are n = t·Hkv + g for both K and V.
    With return_weights, also the softmax weights p [Hq, T]."""
    q = as_f64(q)
    hq = q.shape[0]
    s = rrq.scores(q, k_packed, k_norms, t_len, hkv, d, k_bits, k_seed, k_levels, scale)
    s = s - np.max(s, axis=1, keepdims=True)
    w = np.exp(s)
    p = w / np.sum(w, axis=1, keepdims=True)
    v_hat = rrq.decode_exact(v_packed, v_norms, v_bits, d, v_seed, v_levels).reshape(t_len, hkv, d)
    out = np.empty((hq, d), dtype=np.float64)
    for h in range(hq):
        g = rrq.kv_group(h, hq, hkv)
        out[h] = p[h] @ v_hat[:, g, :]
    return (out, p) if return_weights else out
