"""GPU-vs-oracle parity for rrq_qk_scores_qjl, the unbiased scores on keys stored as
b-bit codes plus the QJL one-bit residual sketch (needs a B200).

The oracle is `oracle.qjl.scores_unbiased`.  Tolerance: each score within
1e-3·|scale| of the sum of the two terms' Cauchy–Schwarz bounds,
‖q_h‖·‖x̂_{t,g}‖ + √(π/2)/d·ρ_{t,g}·‖S·Πq_h‖·√d (a per-element relative error is
undefined near 0), the same 1e-3 that the b-bit scores use.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import qjl as oqjl
from oracle import rng as orng
from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
D = 128


def _s_matrix(seed):
    s = orng.qjl_gaussian(seed, D)  # bf16-exact float64
    return s, torch.from_numpy(s.astype(np.float32)).to(torch.bfloat16).to(DEV)


def _check(q, packed, norms, qbits, rnorm, t_len, hkv, bits, seed, s64, s_dev, scale, what):
    hq = q.shape[0]
    got = B.rrq_qk_scores_qjl(
        torch.from_numpy(q).to(DEV), torch.from_numpy(packed).to(DEV),
        torch.from_numpy(norms.astype(np.float32)).to(DEV), torch.from_numpy(qbits).to(DEV),
        torch.from_numpy(rnorm.astype(np.float32)).to(DEV), s_dev, hkv, D, bits, seed, scale=scale)
    torch.cuda.synchronize()
    got = got.cpu().numpy()
    ref = oqjl.scores_unbiased(q, packed, norms, qbits, rnorm, t_len, hkv, D, bits, seed, s64,
                               scale=scale)
    cs = orc.score_tolerance_scale(q, packed, norms, t_len, hkv, D, bits)
    v = orc.rotate(q.astype(np.float64), seed) @ s64.T  # rows S·Πq_h
    g = np.arange(hq) // (hq // hkv)
    rn = np.asarray(rnorm, np.float64).reshape(t_len, hkv)[:, g].T
    cs = cs + math.sqrt(math.pi / 2) / D * rn * np.linalg.norm(v, axis=1)[:, None] * math.sqrt(D)
    P.assert_scores_close(got, ref, cs, scale, what)
    return got, ref


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("hq,hkv", [(8, 8), (16, 8), (32, 8), (64, 8), (4, 1)])
def test_unbiased_scores_parity_on_oracle_encoded_keys(bits, hq, hkv):
    """Keys encoded by the oracle (MSE codes, QJL bits, norms); several tiles per
    warp plus a ragged tail."""
    rg = np.random.Generator(np.random.PCG64(900 + bits * 10 + hq))
    t_len = 2 * 148 * 8 + 37 if hkv == 1 else 1500
    k = (rg.standard_normal((t_len * hkv, D), dtype=np.float32) * 1.7).astype(np.float16)
    q = rg.standard_normal((hq, D), dtype=np.float32).astype(np.float16)
    s64, s_dev = _s_matrix(4242)
    enc = oqjl.encode(k.astype(np.float64), bits, 42, s64)
    _check(q, enc.enc.packed, enc.enc.norms, enc.bits, enc.rnorm, t_len, hkv, bits, 42, s64, s_dev,
           1.0 / math.sqrt(D), f"b={bits} hq={hq} hkv={hkv}")


def test_unbiased_scores_full_size_sampled():
    """32 query heads against 131072 tokens x 8 kv heads (2-bit codes + QJL bits, the
    TurboQuant split of config 4 on the score workload's shape), with seeded random
    code, bit and norm arrays; sampled tokens checked against the oracle."""
    rg = np.random.Generator(np.random.PCG64(1006))
    t_len, hkv, hq, bits = 131072, 8, 32, 2
    rows = t_len * hkv
    packed = rg.integers(0, 256, size=(rows, D * bits // 8), dtype=np.uint8)
    qbits = rg.integers(0, 256, size=(rows, D // 8), dtype=np.uint8)
    norms = np.exp(rg.standard_normal(rows) * 0.5).astype(np.float32) * 11.0
    rnorm = (norms * rg.uniform(0.2, 0.5, rows)).astype(np.float32)
    q = rg.standard_normal((hq, D), dtype=np.float32).astype(np.float16)
    s64, s_dev = _s_matrix(4242)
    got = B.rrq_qk_scores_qjl(
        torch.from_numpy(q).to(DEV), torch.from_numpy(packed).to(DEV), torch.from_numpy(norms).to(DEV),
        torch.from_numpy(qbits).to(DEV), torch.from_numpy(rnorm).to(DEV), s_dev, hkv, D, bits, 42)
    torch.cuda.synchronize()
    got = got.cpu().numpy()
    toks = np.sort(rg.choice(t_len, 300, replace=False))
    sel = (toks[:, None] * hkv + np.arange(hkv)[None, :]).ravel()
    ref = oqjl.scores_unbiased(q, packed[sel], norms[sel], qbits[sel], rnorm[sel], len(toks), hkv, D,
                               bits, 42, s64)
    cs = orc.score_tolerance_scale(q, packed[sel], norms[sel], len(toks), hkv, D, bits)
    v = orc.rotate(q.astype(np.float64), 42) @ s64.T
    g = np.arange(hq) // (hq // hkv)
    rn = rnorm[sel].astype(np.float64).reshape(len(toks), hkv)[:, g].T
    cs = cs + math.sqrt(math.pi / 2) / D * rn * np.linalg.norm(v, axis=1)[:, None] * math.sqrt(D)
    P.assert_scores_close(got[:, toks], ref, cs, 1.0, "full size sampled")


def test_unbiased_scores_zero_keys_ragged_and_empty():
    rg = np.random.Generator(np.random.PCG64(77))
    hq, hkv, bits = 8, 2, 3
    s64, s_dev = _s_matrix(5)
    for t_len in (1, 31, 33, 95):
        k = rg.standard_normal((t_len * hkv, D)).astype(np.float16)
        k[0] = 0  # a zero key: ν = ρ = 0, score 0
        q = rg.standard_normal((hq, D)).astype(np.float16)
        enc = oqjl.encode(k.astype(np.float64), bits, 9, s64)
        got, _ = _check(q, enc.enc.packed, enc.enc.norms, enc.bits, enc.rnorm, t_len, hkv, bits, 9,
                        s64, s_dev, 1.0, f"T={t_len}")
        assert np.all(got[: hq // hkv, 0] == 0)
    e = B.rrq_qk_scores_qjl(torch.zeros(hq, D, dtype=torch.float16, device=DEV),
                            torch.zeros(0, D * bits // 8, dtype=torch.uint8, device=DEV),
                            torch.zeros(0, dtype=torch.float32, device=DEV),
                            torch.zeros(0, D // 8, dtype=torch.uint8, device=DEV),
                            torch.zeros(0, dtype=torch.float32, device=DEV), s_dev, hkv, D, bits, 9)
    assert e.shape == (hq, 0)


def test_unbiased_scores_from_the_gpu_encoder_reduce_the_bias():
    """End to end on the GPU (rrq_encode with QJL, then the unbiased scores): averaged
    over projections S, the scores approach <q, x> while the 2-bit scores alone stay
    biased low by about D_2 ≈ 0.12 of it (the MSE shrinkage of "Bias vs unbiasedness")."""
    rg = np.random.Generator(np.random.PCG64(31))
    t_len, hkv, bits = 256, 1, 2
    direction = rg.standard_normal(D)
    direction /= np.linalg.norm(direction)
    x = (direction[None, :] * 10.0 + rg.standard_normal((t_len, D)) * 0.3).astype(np.float32)
    q = direction.astype(np.float16)[None]
    xd = torch.from_numpy(x).to(torch.bfloat16).to(DEV)
    truth = xd.double().cpu().numpy() @ q[0].astype(np.float64)
    qd = torch.from_numpy(q).to(DEV)
    acc = np.zeros(t_len)
    n = 64
    for sd in range(n):
        s_dev = B.rrq_qjl_matrix(1000 + sd, D, device=DEV)
        codes, norms, qb, rn = B.rrq_encode(xd, bits, 42, qjl_S=s_dev)
        acc += B.rrq_qk_scores_qjl(qd, codes, norms, qb, rn, s_dev, hkv, D, bits, 42).cpu().numpy()[0]
    mse_only = B.rrq_qk_scores(qd, codes, norms, hkv, D, bits, 42).cpu().numpy()[0]
    bias_mse = np.mean((mse_only - truth) / truth)
    bias_unb = np.mean((acc / n - truth) / truth)
    assert -0.2 < bias_mse < -0.05, bias_mse
    assert abs(bias_unb) < 0.01, bias_unb
