"""Seeded synthetic inputs for the five workloads (shared by tests, bench and smoke).

This module only draws random inputs; it holds none of the quantisation
arithmetic, so the CPU oracle and the CUDA path can both be fed from it.
Every array comes from numpy's PCG64 with a fixed seed.

Workloads (shapes, sizes and distributions as stated for this hot path):

1. ``pr1``     — 4096 fp32 vectors, d = 128, N(0,1) entries except channels
                 {3, 47, 111} scaled ×20; b = 2; seed 1001.
2. ``kv``      — fp16 K cache [32768 tokens × 8 KV heads × 128]: z ~ N(0,1),
                 ⌈2 % · d⌉ = 3 outlier channels per head (drawn once per head,
                 fixed across tokens) scaled ×15, every token scaled by
                 exp(0.5·w_t) with w_t ~ N(0,1) shared across heads
                 (log-normal σ = 0.5); b = 4; seed 1002.
3. ``attnrot`` — fp16 [131072 × 8 × 128], distribution of ``kv``; seed 1003.
4. ``turbo``   — bf16 [1048576 × 128]: N(0,1) with 3 seeded channels drawn
                 from Student-t ν = 3; b = 2 + QJL; seed 1004.
5. ``scores``  — K [131072 × 8 × 128] with the ``kv`` distribution (seed
                 1005), query fp16 [32 × 128] N(0,1); 4-bit codes; scale 1.

The rotation seed is 42 and the QJL seed 4242 throughout.

bf16 inputs are returned as float32 arrays whose values are exactly
representable in bf16 (rounded to nearest even when drawn).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

ROT_SEED = 42
QJL_SEED = 4242


@dataclass
class Workload:
    name: str
    x: np.ndarray                 # [tokens, heads, d] (or [n, d]); float16 / float32
    dtype: str                    # 'f16' | 'bf16' | 'f32' (the input element type)
    bits: int
    seed: int = ROT_SEED
    extra: dict = field(default_factory=dict)

    @property
    def d(self) -> int:
        return self.x.shape[-1]

    @property
    def n(self) -> int:
        return int(np.prod(self.x.shape[:-1]))

    def flat(self) -> np.ndarray:
        return self.x.reshape(self.n, self.d)


def to_bf16_exact(a: np.ndarray) -> np.ndarray:
    """float32 array -> float32 array of the nearest bf16 values (ties to even)."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16) << 16
    return (rounded & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def _kv_like(rng: np.random.Generator, tokens: int, heads: int, d: int) -> np.ndarray:
    k = math.ceil(0.02 * d)
    z = rng.standard_normal((tokens, heads, d), dtype=np.float32)
    gain = np.ones((heads, d), dtype=np.float32)
    for h in range(heads):
        gain[h, rng.choice(d, k, replace=False)] = 15.0
    w = rng.standard_normal(tokens).astype(np.float32)
    tok = np.exp(0.5 * w).astype(np.float32)
    return z * gain[None] * tok[:, None, None]


def pr1(n: int = 4096, d: int = 128) -> Workload:
    rng = np.random.Generator(np.random.PCG64(1001))
    x = rng.standard_normal((n, d), dtype=np.float32)
    ch = [c for c in (3, 47, 111) if c < d]
    x[:, ch] *= 20.0
    return Workload("pr1", x, "f32", 2, extra={"outlier_channels": ch})


def kv(tokens: int = 32768, heads: int = 8, d: int = 128, bits: int = 4, seed: int = 1002) -> Workload:
    rng = np.random.Generator(np.random.PCG64(seed))
    x = _kv_like(rng, tokens, heads, d).astype(np.float16)
    return Workload("kv", x, "f16", bits)


def attnrot(tokens: int = 131072, heads: int = 8, d: int = 128) -> Workload:
    rng = np.random.Generator(np.random.PCG64(1003))
    x = _kv_like(rng, tokens, heads, d).astype(np.float16)
    return Workload("attnrot", x, "f16", 4)


def turbo(n: int = 1048576, d: int = 128) -> Workload:
    rng = np.random.Generator(np.random.PCG64(1004))
    x = rng.standard_normal((n, d), dtype=np.float32)
    ch = rng.choice(d, 3, replace=False)
    x[:, ch] = rng.standard_t(3.0, size=(n, 3)).astype(np.float32)
    return Workload("turbo", to_bf16_exact(x), "bf16", 2,
                    extra={"heavy_channels": [int(c) for c in ch], "qjl_seed": QJL_SEED})


def scores(tokens: int = 131072, hkv: int = 8, hq: int = 32, d: int = 128, bits: int = 4) -> Workload:
    rng = np.random.Generator(np.random.PCG64(1005))
    k = _kv_like(rng, tokens, hkv, d).astype(np.float16)
    q = rng.standard_normal((hq, d), dtype=np.float32).astype(np.float16)
    return Workload("scores", k, "f16", bits, extra={"q": q, "hq": hq, "hkv": hkv, "scale": 1.0})


def gaussian(n: int, d: int, dtype: str = "f16", seed: int = 7, scale: float = 1.0) -> Workload:
    """Plain N(0, scale²) vectors, for sweeps and edge cases."""
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((n, d), dtype=np.float32) * np.float32(scale)
    if dtype == "f16":
        x = x.astype(np.float16)
    elif dtype == "bf16":
        x = to_bf16_exact(x)
    return Workload("gaussian", x, dtype, 4)


CONFIGS = {
    1: ("pr1", "4096 fp32 vectors d=128, 3 outlier channels x20, b=2"),
    2: ("kv", "fp16 KV [32768 x 8 x 128], 2% outlier channels x15, log-normal token scale, b=4"),
    3: ("attnrot", "fp16 K [131072 x 8 x 128], kv distribution, RHT + q4_0"),
    4: ("turbo", "bf16 [1048576 x 128], 3 Student-t(3) channels, b=2 + QJL"),
    5: ("scores", "scores: 32 q heads, 8 KV heads, 131072 keys d=128 at b=4"),
}
