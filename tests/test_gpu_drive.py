"""GPU-vs-oracle parity for DRIVE's one-bit encoder (rrq_drive_encode), and for
its decodes through the one-bit decoder and score path (needs a B200).

"Random-rotation quantization" page, "History", DRIVE bullet and "Three
decoders, one rotation", mean decoder.  The oracle is `oracle.sphere`.

Tolerances:
* sign bits: exact, except where the oracle's normalised coordinate
  u = √d·(Πx)_i/‖x‖ lies within 1e-5 of 0 (the encoder's own exemption band);
* the stored scale S·√d: relative error ≤ (d·log₂d + 2d + 4)·2⁻²⁴, the worst
  case of the fp32 arithmetic: every unnormalised rotated coordinate y'_i takes
  log₂d roundings of partial sums bounded by ‖x‖₁ ≤ ‖y'‖₁, the L1 and squared
  norm sums take d roundings each, and the final product and quotient one each;
* reconstructions and scores: the encode/decode tolerances of tests/parity.py
  (2e-3·‖x‖ and 1e-3·‖q‖·‖x̂‖, with ‖x̂‖ = S·√d).
Rows where a sign differs inside the exemption band are decoded from the
oracle's bits (one flipped sign moves x̂ by 2S, far outside 2e-3·‖x‖).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import hadamard
from oracle import rrq as orc
from oracle import sphere
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SIGNS = [-1.0, 1.0]


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)  # values are bf16-exact
    return t.to(DEV)


def scale_tol(d: int) -> float:
    return (d * math.log2(d) + 2 * d + 4) * 2.0 ** -24


def gpu_drive(x: np.ndarray, dtype: str, seed: int, unbiased: bool):
    codes, scales = B.rrq_drive_encode(to_dev(x, dtype), seed, unbiased)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def check_drive(x: np.ndarray, dtype: str, seed: int, unbiased: bool, what: str):
    """Encode on the GPU and check bits and scales; returns (oracle, packed bits
    with exempt rows taken from the oracle, GPU scales)."""
    d = x.shape[-1]
    x64 = x.astype(np.float64)
    enc = sphere.drive_encode(x64, seed, unbiased)
    codes, scales = gpu_drive(x, dtype, seed, unbiased)
    nrm = np.linalg.norm(x64, axis=1)
    u = math.sqrt(d) * enc.rx / np.where(nrm > 0, nrm, 1.0)[:, None]
    bits = P.unpack_codes(codes, 1, d)
    P.assert_codes_match(bits, enc.signs, u, np.array([0.0]), what)
    bad_rows = np.any(bits != enc.signs, axis=1)
    packed = codes.reshape(enc.packed.shape).copy()
    packed[bad_rows] = enc.packed[bad_rows]
    ref = enc.scale * math.sqrt(d)
    rel = np.abs(scales.astype(np.float64) - ref) / np.maximum(ref, 1e-300)
    rel[ref == 0] = np.abs(scales[ref == 0])
    assert np.all(rel <= scale_tol(d)), f"{what}: scale relative error {rel.max()} > {scale_tol(d)}"
    return enc, packed, scales


@pytest.mark.parametrize("unbiased", [False, True])
@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
def test_drive_encode_and_mean_decoder(d, dtype, unbiased):
    # 16-bit rows with d <= 128 take the batch encoder: several rounds of its
    # 148-CTA x 8-warp x 32-row grid plus a ragged tail
    n = 148 * 8 * 32 * 2 + 19 if d <= 128 else 3001
    x = W.gaussian(n, d, dtype, seed=d * 7 + len(dtype) + int(unbiased), scale=1.9).flat()
    seed = 0x5EED + d
    what = f"drive d={d} {dtype} unbiased={unbiased}"
    enc, packed, scales = check_drive(x, dtype, seed, unbiased, what)
    # x̂ = S·Πᵀ·sign(Πx), through the one-bit decoder with the ±1 codebook
    rows = np.arange(0, n, 7) if n > 20000 else np.arange(n)
    pc = torch.from_numpy(packed).to(DEV)
    sc = torch.from_numpy(scales).to(DEV)
    xh = B.rrq_decode(pc, sc, d, 1, seed, codebook=SIGNS, out_dtype=torch.float32)
    torch.cuda.synchronize()
    xh = xh.cpu().numpy().astype(np.float64)[rows]
    p = hadamard.rotation_matrix(seed, d)
    # the oracle's bits: a coordinate with (Πx)_i = 0 exactly (common for
    # bf16 inputs) decodes to −1 on both sides
    ref = sphere.drive_mean_decode(p, enc.signs[rows], enc.scale[rows])
    xs = np.linalg.norm(x[rows].astype(np.float64), axis=1)
    P.assert_reconstruction_close(xh, ref, xs, what)


@pytest.mark.parametrize("unbiased", [False, True])
@pytest.mark.parametrize("d", [64, 128])
def test_drive_scores_are_scale_times_sign_inner_product(d, unbiased):
    """rrq_qk_scores over DRIVE bits: scale·S·⟨Πq, sign(Πx)⟩ per (head, token)."""
    hq, hkv, T = 32, 8, 2 * 148 * 32 + 5
    rng = np.random.Generator(np.random.PCG64(400 + d))
    k = (rng.standard_normal((T, hkv, d), dtype=np.float32) * 2.2).astype(np.float16)
    q = rng.standard_normal((hq, d), dtype=np.float32).astype(np.float16)
    seed, scale = 77 + d, 1.0 / math.sqrt(d)
    enc, packed, scales = check_drive(k.reshape(T * hkv, d), "f16", seed, unbiased, f"scores d={d}")
    s = B.rrq_qk_scores(torch.from_numpy(q).to(DEV), torch.from_numpy(packed).to(DEV),
                        torch.from_numpy(scales).to(DEV), hkv, d, 1, seed, codebook=SIGNS,
                        scale=scale)
    torch.cuda.synchronize()
    s = s.cpu().numpy()
    bits = orc.unpack_codes(packed, 1, d).reshape(T, hkv, d)
    qr = orc.rotate(q.astype(np.float64), seed)  # Πq
    S = enc.scale.reshape(T, hkv)
    g = np.arange(hq) // (hq // hkv)
    ref = scale * S[:, g].T * np.einsum("hi,thi->ht", qr, 2.0 * bits[:, g, :] - 1.0)
    cs = np.linalg.norm(q.astype(np.float64), axis=1)[:, None] * (S[:, g].T * math.sqrt(d))
    P.assert_scores_close(s, ref, cs, scale, f"drive scores d={d} unbiased={unbiased}")


@pytest.mark.parametrize("unbiased", [False, True])
@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_drive_zero_rows_ragged_and_empty(dtype, unbiased):
    """x = 0 gives all-zero bits and a zero scale in both modes; n = 0 is a no-op."""
    d = 128
    x = W.gaussian(1000, d, dtype, seed=5, scale=3.0).flat().copy()
    x[[0, 17, 999]] = 0
    x[500] = x[500] * np.asarray(1000.0, x.dtype)  # a large row
    enc, packed, scales = check_drive(x, dtype, 3, unbiased, f"edge {dtype}")
    assert np.all(packed[[0, 17, 999]] == 0) and np.all(scales[[0, 17, 999]] == 0)
    for n in (1, 31, 33):
        check_drive(x[1:1 + n], dtype, 3, unbiased, f"n={n}")
    codes, scales = B.rrq_drive_encode(torch.empty(0, d, dtype=torch.float16, device=DEV), 3, unbiased)
    assert codes.shape == (0, d // 8) and scales.shape == (0,)


def test_drive_unbiased_inner_product_is_exact_for_x_itself():
    """The unbiased scale makes ⟨x̂, x⟩ = ‖x‖² for every vector (with S from the
    GPU's stored value: ⟨S·Πᵀsign(Πx), x⟩ = S·‖Πx‖₁)."""
    d = 128
    x = W.gaussian(4096, d, "bf16", seed=11, scale=0.7).flat()
    enc, packed, scales = check_drive(x, "bf16", 19, True, "unbiased ip")
    x64 = x.astype(np.float64)
    xh = B.rrq_decode(torch.from_numpy(packed).to(DEV), torch.from_numpy(scales).to(DEV), d, 1, 19,
                      codebook=SIGNS, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ip = np.sum(xh.cpu().numpy().astype(np.float64) * x64, axis=1)
    nn = np.sum(x64 * x64, axis=1)
    assert np.all(np.abs(ip - nn) <= 1e-5 * nn)
