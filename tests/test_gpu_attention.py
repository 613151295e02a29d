"""GPU-vs-oracle parity for rrq_attention_decode, one decode step of attention over a
quantised K/V cache (needs a B200).

The oracle is `oracle.attention.decode_attention`.  Tolerance, per query head h:

    ‖out_gpu[h] − out_oracle[h]‖ ≤ 2e-3 · Σ_t p[h,t]·‖v̂_{t,g(h)}‖,

with p the oracle's softmax weights.  The output is the convex combination
Σ_t p[h,t]·v̂_t; if every term carries at most the reconstruction tolerance
(2e-3 relative) then, by the triangle inequality, so does the sum, against the
weighted sum of the reconstruction norms.  The kernel's own rounding stays well
inside it: fp16 levels and weights (2⁻¹² relative each, fp32 accumulation) and
the fp16 score operands, whose error moves every weight p by a relative
≈ |scale|·‖q‖·ν^K·2⁻¹¹/√d (below 1e-3 for the workloads here).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B
from tests.parity import attention_bound as weighted_bound

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
D = 128
REL = 2e-3  # the reconstruction tolerance


def _run(q, kp, kn, vp, vn, hkv, ks, vs, scale, d=D, kb=4, vb=4):
    out = B.rrq_attention_decode(
        torch.from_numpy(q).to(DEV), torch.from_numpy(kp).to(DEV),
        torch.from_numpy(kn.astype(np.float32)).to(DEV), torch.from_numpy(vp).to(DEV),
        torch.from_numpy(vn.astype(np.float32)).to(DEV), hkv, d, ks, vs, scale=scale,
        k_bits=kb, v_bits=vb)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check(q, kp, kn, vp, vn, t_len, hkv, ks, vs, scale, what, d=D, kb=4, vb=4):
    got = _run(q, kp, kn, vp, vn, hkv, ks, vs, scale, d, kb, vb)
    ref, p = oatt.decode_attention(q, kp, kn, vp, vn, t_len, hkv, d, kb, vb, ks, vs, scale=scale,
                                   return_weights=True)
    bound = weighted_bound(p, vp, vn, t_len, hkv, d, vb, vs)
    err = np.linalg.norm(got - ref, axis=1)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    assert np.all(err <= bound), f"{what}: worst error/bound {np.max(err / bound)}"
    return got, ref


def _cache(rg, t_len, hkv, ks, vs, d=D, kb=4, vb=4):
    k = (rg.standard_normal((t_len * hkv, d)) * 1.5).astype(np.float16).astype(np.float64)
    v = (rg.standard_normal((t_len * hkv, d)) * 0.8).astype(np.float16).astype(np.float64)
    ek, ev = orc.encode(k, kb, ks), orc.encode(v, vb, vs)
    return ek.packed, ek.norms, ev.packed, ev.norms


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (4, 1), (2, 2)])
@pytest.mark.parametrize("t_len", [1, 37, 2000])
def test_attention_parity_on_oracle_encoded_cache(hq, hkv, t_len):
    rg = np.random.Generator(np.random.PCG64(hq * 1000 + hkv * 10 + t_len))
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 42, 43)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 42, 43, 1.0 / math.sqrt(D), f"hq={hq} hkv={hkv} T={t_len}")


@pytest.mark.parametrize("d,kb,vb", [(128, 2, 2), (128, 3, 3), (64, 4, 4), (256, 4, 4), (128, 4, 2),
                                     (64, 1, 3), (512, 2, 4), (256, 3, 1)])
@pytest.mark.parametrize("hq,hkv", [(32, 8), (4, 1), (16, 2)])
@pytest.mark.parametrize("t_len", [1, 37, 2000])
def test_attention_general_shapes(d, kb, vb, hq, hkv, t_len):
    """Every shape other than d = 128 with 4-bit K and V (the scores through the score
    kernel into the workspace, then the fp32 value sums): the same per-head bound."""
    if d == 512 and hq // hkv == 8:
        pytest.skip("d = 512 takes groups of at most 4")
    rg = np.random.Generator(np.random.PCG64(d * 100 + kb * 10 + vb + hq + 7 * t_len))
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 42, 43, d, kb, vb)
    q = rg.standard_normal((hq, d)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 42, 43, 1.0 / math.sqrt(d), f"d={d} b={kb}/{vb} hq={hq} hkv={hkv} T={t_len}",
           d, kb, vb)


def test_attention_general_value_norm_range():
    """The general path sums in fp32: value norms from 1e-30 to 1e30 keep the bound."""
    rg = np.random.Generator(np.random.PCG64(71))
    hq, hkv, t_len, d = 8, 2, 500, 64
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 42, 43, d, 2, 3)
    q = rg.standard_normal((hq, d)).astype(np.float16)
    for v_scale in (1e-30, 1e30):
        vs = (vn * v_scale * np.exp(rg.standard_normal(vn.shape))).astype(np.float32)
        _check(q, kp, kn, vp, vs, t_len, hkv, 42, 43, 0.125, f"general v scale {v_scale}", d, 2, 3)


def test_attention_special_cases():
    """One token returns its value; a zero query averages the values; a large scale
    picks the top-scoring token's value.  Each is held to the reconstruction
    tolerance against the exact answer as well as against the oracle."""
    rg = np.random.Generator(np.random.PCG64(5))
    hq, hkv = 4, 2
    kp, kn, vp, vn = _cache(rg, 1, hkv, 7, 8)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    got, _ = _check(q, kp, kn, vp, vn, 1, hkv, 7, 8, 1.0, "one token")
    v_hat = orc.decode_exact(vp, vn, 4, D, 8)
    want = v_hat[np.arange(hq) // 2]
    assert np.all(np.linalg.norm(got - want, axis=1) <= REL * np.linalg.norm(want, axis=1))
    t_len = 300
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 7, 8)
    got, _ = _check(np.zeros((hq, D), np.float16), kp, kn, vp, vn, t_len, hkv, 7, 8, 1.0, "zero query")
    v_hat = orc.decode_exact(vp, vn, 4, D, 8).reshape(t_len, hkv, D)
    for h in range(hq):
        g = h // 2
        want = v_hat[:, g].mean(axis=0)
        assert np.linalg.norm(got[h] - want) <= REL * np.linalg.norm(v_hat[:, g], axis=1).mean()
    q = rg.standard_normal((hq, D)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 7, 8, 50.0, "large scale")


@pytest.mark.parametrize("v_scale", [1e-7, 1e-4, 3e3, 1e6])
def test_attention_value_norm_range(v_scale):
    """Value norms far from 1 (tiny and huge): the weights p·ν^V must neither flush to
    zero nor overflow in the value product, so the relative tolerance holds at any
    scale of the value cache."""
    rg = np.random.Generator(np.random.PCG64(int(abs(math.log10(v_scale))) + 17))
    hq, hkv, t_len = 16, 4, 700
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 42, 43)
    # a vector scaled by c keeps its codes and has norm c·ν; spread the norms over
    # several orders of magnitude within the cache, too
    vn = (vn * v_scale * np.exp(rg.standard_normal(vn.shape) * 2.0)).astype(np.float32)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 42, 43, 1.0 / math.sqrt(D), f"v scale {v_scale}")


def test_attention_full_size_sampled_group():
    """32 query heads over 131072 tokens x 8 kv heads (the score workload's shape), with
    seeded random codes and norms; the oracle checks two kv heads' groups on their own
    slices of the cache (the other groups share nothing with them)."""
    rg = np.random.Generator(np.random.PCG64(1007))
    t_len, hkv, hq = 131072, 8, 32
    rows = t_len * hkv
    kp = rg.integers(0, 256, size=(rows, 64), dtype=np.uint8)
    vp = rg.integers(0, 256, size=(rows, 64), dtype=np.uint8)
    kn = (np.exp(rg.standard_normal(rows) * 0.5) * 11.0).astype(np.float32)
    vn = (np.exp(rg.standard_normal(rows) * 0.5) * 9.0).astype(np.float32)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    scale = 1.0 / math.sqrt(D)
    got = _run(q, kp, kn, vp, vn, hkv, 42, 43, scale)
    assert np.all(np.isfinite(got))
    for g in (0, 5):
        sel = np.arange(t_len) * hkv + g
        heads = np.arange(g * 4, g * 4 + 4)
        ref, p = oatt.decode_attention(q[heads], kp[sel], kn[sel], vp[sel], vn[sel], t_len, 1, D, 4,
                                       4, 42, 43, scale=scale, return_weights=True)
        bound = weighted_bound(p, vp[sel], vn[sel], t_len, 1, D, 4, 43)
        assert np.all(bound <= 5e-3 * np.linalg.norm(ref, axis=1))  # the bound is a tight one
        err = np.linalg.norm(got[heads] - ref, axis=1)
        assert np.all(err <= bound), (g, np.max(err / bound))
