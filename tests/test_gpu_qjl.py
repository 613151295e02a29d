"""GPU-vs-oracle parity for rrq_encode with the QJL residual sketch (tcgen05; needs a B200).

Codes and norms follow the encode rules.  For every vector whose codes match
the oracle's, the residual norm must agree to 1e-4 (relative) and every sign
bit must agree except where the oracle's projection |v_i| < 1e-5·ρ; such
exempt bits must be fewer than 1e-4 of all bits.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import codebook as ocb
from oracle import qjl as oqjl
from oracle import rng as orng
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)
    return t.to(DEV)


_S_CACHE = {}


def s_matrix(seed=4242, d=128):
    if (seed, d) not in _S_CACHE:
        _S_CACHE[(seed, d)] = orng.qjl_gaussian(seed, d)
    return _S_CACHE[(seed, d)]


def check_qjl(x, dtype, bits, what, codebook=None):
    d = x.shape[1]
    s_dev = B.rrq_qjl_matrix(4242, d, device=DEV)
    codes, norms, qb, rn = B.rrq_encode(to_dev(x, dtype), bits, 42, codebook=codebook, qjl_S=s_dev)
    torch.cuda.synchronize()
    codes, norms, qb, rn = (t.cpu().numpy() for t in (codes, norms, qb, rn))
    levels = None if codebook is None else np.asarray(codebook, np.float64)
    enc = oqjl.encode(x.astype(np.float64), bits, 42, s_matrix(4242, d), levels)
    tau = ocb.thresholds(ocb.lloyd_max(bits) if levels is None else levels)
    gc = P.unpack_codes(codes, bits, d)
    P.assert_codes_match(gc, enc.enc.codes, enc.enc.u, tau, what)
    P.assert_norms_close(norms, enc.enc.norm64, d, what)
    assert np.all(np.isfinite(rn)), f"{what}: a tensor-core stage timed out (NaN residual norm)"
    same = np.all(gc == enc.enc.codes, axis=1)  # norms may differ by an ulp (r moves ~1e-7·ρ)
    assert same.mean() > 0.99
    rho = enc.rnorm.astype(np.float64)
    rel = np.abs(rn[same] - rho[same]) / np.maximum(rho[same], 1e-30)
    assert np.all(rel <= 1e-4), f"{what}: residual norm error {rel.max()}"
    gb = np.unpackbits(qb[same], axis=1, bitorder="little")[:, :d]
    ob = np.unpackbits(enc.bits[same], axis=1, bitorder="little")[:, :d]
    diff = gb != ob
    near = np.abs(enc.v[same]) < 1e-5 * rho[same, None]
    assert not np.any(diff & ~near), f"{what}: {int(np.sum(diff & ~near))} sign bits differ outside the band"
    assert diff.sum() < 1e-4 * diff.size + 1, f"{what}: {int(diff.sum())} exempt sign bits"
    return enc


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_qjl_parity_turbo_distribution(bits):
    w = W.turbo(n=1000)
    check_qjl(w.flat(), "bf16", bits, f"qjl b={bits}")


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_qjl_parity_other_dtypes(dtype):
    x = W.gaussian(700, 128, dtype, seed=3, scale=2.0).flat()
    check_qjl(x, dtype, 2, f"qjl {dtype}")


@pytest.mark.parametrize("n", [1, 127, 128, 129, 300])
def test_qjl_ragged_tiles(n):
    x = W.turbo(n=max(n, 1)).flat()[:n]
    check_qjl(x, "bf16", 2, f"qjl n={n}")


def test_qjl_custom_asymmetric_codebook():
    cb = np.sort(np.random.default_rng(8).normal(size=4)).astype(np.float32)
    check_qjl(W.turbo(n=400).flat(), "bf16", 2, "qjl asym", codebook=cb)


def test_qjl_codes_equal_plain_encode():
    """The fused QJL kernel writes the same codes as the plain encoder (norms: summation order)."""
    x = to_dev(W.turbo(n=2048).flat(), "bf16")
    s_dev = B.rrq_qjl_matrix(4242, 128, device=DEV)
    c1, n1, _, _ = B.rrq_encode(x, 2, 42, qjl_S=s_dev)
    c2, n2 = B.rrq_encode(x, 2, 42)
    torch.cuda.synchronize()
    assert torch.equal(c1, c2)
    assert torch.all((n1 - n2).abs() <= 128 * 2.0 ** -24 * n2)


def test_qjl_full_size_sampled():
    """Workload 4: 1,048,576 bf16 vectors in one launch; 2000 sampled rows (plus the
    first and the last) held to the same rules as the small cases: codes with the
    boundary exemption, norms to fp32 summation order, residual norms to 1e-4 and
    sign bits outside the 1e-5·ρ band, with the exempt bits under 1e-4."""
    w = W.turbo()
    x = w.flat()
    xd = to_dev(x, "bf16")
    s_dev = B.rrq_qjl_matrix(4242, 128, device=DEV)
    codes, norms, qb, rn = B.rrq_encode(xd, 2, 42, qjl_S=s_dev)
    torch.cuda.synchronize()
    assert torch.all(torch.isfinite(rn)), "a tensor-core stage timed out (NaN residual norm)"
    rows = np.sort(np.random.default_rng(4).choice(x.shape[0], 2000, replace=False))
    rows = np.concatenate([[0], rows, [x.shape[0] - 1]])
    r_t = torch.from_numpy(rows).to(DEV)
    enc = oqjl.encode(x[rows].astype(np.float64), 2, 42, s_matrix())
    tau = ocb.thresholds(ocb.lloyd_max(2))
    gc = P.unpack_codes(codes[r_t].cpu().numpy(), 2, 128)
    P.assert_codes_match(gc, enc.enc.codes, enc.enc.u, tau, "qjl full size")
    P.assert_norms_close(norms[r_t].cpu().numpy(), enc.enc.norm64, 128, "qjl full size")
    same = np.all(gc == enc.enc.codes, axis=1)
    assert same.mean() > 0.99
    rho = enc.rnorm.astype(np.float64)
    rn_s = rn[r_t].cpu().numpy().astype(np.float64)
    rel = np.abs(rn_s[same] - rho[same]) / np.maximum(rho[same], 1e-30)
    assert np.all(rel <= 1e-4), f"residual norm error {rel.max()}"
    gb = np.unpackbits(qb[r_t].cpu().numpy()[same], axis=1, bitorder="little")
    ob = np.unpackbits(enc.bits[same], axis=1, bitorder="little")
    diff = gb != ob
    near = np.abs(enc.v[same]) < 1e-5 * rho[same, None]
    assert not np.any(diff & ~near), f"{int(np.sum(diff & ~near))} sign bits differ outside the band"
    assert diff.sum() < 1e-4 * diff.size + 1, f"{int(diff.sum())} exempt sign bits"


def test_qjl_estimator_reduces_inner_product_bias():
    """Residual chain: <q, x̂> + √(π/2)/d·ρ·<SΠq, sign> is unbiased where <q, x̂> is shrunk."""
    from oracle import rrq as orc
    w = W.turbo(n=20000)
    x = w.flat()
    s_dev = B.rrq_qjl_matrix(4242, 128, device=DEV)
    codes, norms, qb, rn = B.rrq_encode(to_dev(x, "bf16"), 2, 42, qjl_S=s_dev)
    xh = B.rrq_decode(codes, norms, 128, 2, 42, out_dtype=torch.float32).double().cpu().numpy()
    torch.cuda.synchronize()
    x64 = x.astype(np.float64)
    q = x64 + np.random.default_rng(0).standard_normal(x64.shape)  # correlated queries
    ip = np.sum(q * x64, 1)
    mse = np.sum(q * xh, 1)
    qr = orc.rotate(q, 42)
    corr = np.array([oqjl.estimate_residual_dot(qr[i], s_matrix(), qb[i:i + 1].cpu().numpy(),
                                                rn[i:i + 1].cpu().numpy())[0] for i in range(2000)])
    bias_mse = np.mean(mse[:2000] - ip[:2000])
    bias_prod = np.mean(mse[:2000] + corr - ip[:2000])
    assert bias_mse < 0 and abs(bias_prod) < 0.25 * abs(bias_mse)


def test_qjl_unsupported_head_dim():
    x = torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV)
    s = torch.zeros(64, 64, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(B.RRQError) as e:
        B.rrq_encode(x, 2, 42, qjl_S=s)
    assert e.value.status == B.RRQ_ERR_UNSUPPORTED
