"""GPU-vs-oracle parity for rrq_attention_decode, one decode step of attention over a
4-bit K/V cache (needs a B200).

The oracle is `oracle.attention.decode_attention`.  Tolerance: per head,
‖out_gpu − out_oracle‖ ≤ 2e-3·max_t ‖v̂_{t,g}‖ — the reconstruction tolerance of the
MSE decoder, applied to the convex combination of reconstructions that the output
is (the scores' own fp16 error moves the softmax weights far less).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
D = 128


def _run(q, kp, kn, vp, vn, hkv, ks, vs, scale):
    out = B.rrq_attention_decode(
        torch.from_numpy(q).to(DEV), torch.from_numpy(kp).to(DEV),
        torch.from_numpy(kn.astype(np.float32)).to(DEV), torch.from_numpy(vp).to(DEV),
        torch.from_numpy(vn.astype(np.float32)).to(DEV), hkv, D, ks, vs, scale=scale)
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def _check(q, kp, kn, vp, vn, t_len, hkv, ks, vs, scale, what):
    got = _run(q, kp, kn, vp, vn, hkv, ks, vs, scale)
    ref = oatt.decode_attention(q, kp, kn, vp, vn, t_len, hkv, D, 4, 4, ks, vs, scale=scale)
    vn_max = np.asarray(vn, np.float64).reshape(t_len, hkv).max(axis=0)  # ‖v̂‖ ≤ ν·max|c|/√d·√d
    cmax = np.max(np.abs(orc.default_levels(4)))
    g = np.arange(q.shape[0]) // (q.shape[0] // hkv)
    bound = 2e-3 * vn_max[g] * cmax
    err = np.linalg.norm(got - ref, axis=1)
    assert np.all(err <= bound), f"{what}: error {err.max()} vs bound {bound.min()}"
    return got, ref


def _cache(rg, t_len, hkv, ks, vs):
    k = (rg.standard_normal((t_len * hkv, D)) * 1.5).astype(np.float16).astype(np.float64)
    v = (rg.standard_normal((t_len * hkv, D)) * 0.8).astype(np.float16).astype(np.float64)
    ek, ev = orc.encode(k, 4, ks), orc.encode(v, 4, vs)
    return ek.packed, ek.norms, ev.packed, ev.norms


@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (4, 1), (2, 2)])
@pytest.mark.parametrize("t_len", [1, 37, 2000])
def test_attention_parity_on_oracle_encoded_cache(hq, hkv, t_len):
    rg = np.random.Generator(np.random.PCG64(hq * 1000 + hkv * 10 + t_len))
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 42, 43)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 42, 43, 1.0 / math.sqrt(D), f"hq={hq} hkv={hkv} T={t_len}")


def test_attention_special_cases():
    """One token returns its value; a zero query averages the values; a large scale
    picks the top-scoring token's value.  The weighted sum runs on fp16 levels and
    weights (fp32 accumulation), so the value checks use the reconstruction
    tolerance, 2e-3 of the largest |v̂|."""
    rg = np.random.Generator(np.random.PCG64(5))
    hq, hkv = 4, 2
    kp, kn, vp, vn = _cache(rg, 1, hkv, 7, 8)
    q = rg.standard_normal((hq, D)).astype(np.float16)
    got, _ = _check(q, kp, kn, vp, vn, 1, hkv, 7, 8, 1.0, "one token")
    v_hat = orc.decode_exact(vp, vn, 4, D, 8)
    # fp16 level and weight operands: within the reconstruction tolerance (2e-3 relative)
    assert np.allclose(got, v_hat[np.arange(hq) // 2], atol=2e-3 * np.abs(v_hat).max())
    t_len = 300
    kp, kn, vp, vn = _cache(rg, t_len, hkv, 7, 8)
    got, _ = _check(np.zeros((hq, D), np.float16), kp, kn, vp, vn, t_len, hkv, 7, 8, 1.0, "zero query")
    v_hat = orc.decode_exact(vp, vn, 4, D, 8).reshape(t_len, hkv, D)
    assert np.allclose(got[0], v_hat[:, 0].mean(axis=0), atol=2e-3 * np.abs(v_hat[:, 0]).max())
    q = rg.standard_normal((hq, D)).astype(np.float16)
    _check(q, kp, kn, vp, vn, t_len, hkv, 7, 8, 50.0, "large scale")


def test_attention_full_size_sampled_group():
    """32 query heads over 131072 tokens x 8 kv heads (the score workload's shape), with
    seeded random codes and norms; the oracle checks one kv head's group on its own
    slice of the cache (the other groups share nothing with it)."""
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
    for g in (0, 5):
        sel = np.arange(t_len) * hkv + g
        heads = np.arange(g * 4, g * 4 + 4)
        ref = oatt.decode_attention(q[heads], kp[sel], kn[sel], vp[sel], vn[sel], t_len, 1, D, 4, 4,
                                    42, 43, scale=scale)
        bound = 2e-3 * float(vn[sel].max()) * float(np.max(np.abs(orc.default_levels(4))))
        err = np.linalg.norm(got[heads] - ref, axis=1)
        assert np.all(err <= bound), (g, err.max(), bound)
