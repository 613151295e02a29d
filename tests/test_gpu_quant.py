"""GPU-vs-oracle parity for rotate / encode / decode through the C ABI (needs a B200).

Inputs come from the seeded generators; the oracle runs on the same values.
Sizes span several blocks of the grid-stride loop plus a ragged tail.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import codebook as ocb
from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)  # values are bf16-exact
    return t.to(DEV)


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def run_encode(x_np, dtype, bits, seed, codebook=None):
    xd = to_dev(x_np, dtype)
    codes, norms = B.rrq_encode(xd, bits, seed, codebook=codebook)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), norms.cpu().numpy()


def check_encode(x_np, dtype, bits, seed=42, codebook=None, what=""):
    d = x_np.shape[-1]
    codes, norms = run_encode(x_np, dtype, bits, seed, codebook)
    levels = None if codebook is None else np.asarray(codebook, np.float64)
    enc = orc.encode(x_np.astype(np.float64), bits, seed, levels)
    tau = ocb.thresholds(ocb.lloyd_max(bits) if levels is None else levels)
    gpu_codes = P.unpack_codes(codes, bits, d)
    exempt = P.assert_codes_match(gpu_codes, enc.codes, enc.u, tau, what)
    if exempt == 0:
        assert np.array_equal(codes.reshape(enc.packed.shape), enc.packed), what
    P.assert_norms_close(norms, enc.norm64, d, what)
    return enc, codes, norms


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("inverse", [False, True])
def test_rotate_parity(dtype, d, inverse):
    w = W.gaussian(1037, d, dtype, seed=d + 3, scale=3.0)
    x = w.flat()
    y = B.rrq_rotate(to_dev(x, dtype), 42, inverse=inverse)
    torch.cuda.synchronize()
    ref = orc.rotate(x.astype(np.float64), 42, inverse=inverse)
    P.assert_rotated_close(host_f64(y), ref, np.linalg.norm(x.astype(np.float64), axis=1),
                           f"rotate {dtype} d={d} inv={inverse}")


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_encode_parity(dtype, d, bits):
    w = W.gaussian(777, d, dtype, seed=bits * 1000 + d, scale=2.0)
    check_encode(w.flat(), dtype, bits, what=f"encode {dtype} d={d} b={bits}")


@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_decode_parity_on_oracle_codes(out_dtype, d, bits):
    """The GPU decodes the oracle's codes and norms; compare reconstructions."""
    x = W.gaussian(555, d, "f32", seed=bits * 77 + d, scale=1.5).flat().astype(np.float64)
    enc = orc.encode(x, bits, 42)
    codes = torch.from_numpy(enc.packed).to(DEV)
    norms = torch.from_numpy(enc.norms).to(DEV)
    out = B.rrq_decode(codes, norms, d, bits, 42, out_dtype=TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    ref = orc.decode(enc.packed, enc.norms, bits, d, 42, out_dtype=out_dtype)
    xn = np.linalg.norm(x, axis=1)
    P.assert_reconstruction_close(host_f64(out), ref, xn, f"decode {out_dtype} d={d} b={bits}")
    if out_dtype == "f32":
        exact = orc.decode_exact(enc.packed, enc.norms, bits, d, 42)
        P.assert_rotated_close(host_f64(out), exact, xn, "decode f32 tight")


def test_kv_workload_encode_decode_parity():
    """Workload 2 distribution (outlier channels, log-normal token scale), b = 4, fp16."""
    w = W.kv(tokens=640)
    x = w.flat()
    enc, codes, norms = check_encode(x, "f16", 4, what="kv")
    out = B.rrq_decode(torch.from_numpy(enc.packed).to(DEV), torch.from_numpy(enc.norms).to(DEV),
                       128, 4, 42, out_dtype=torch.float16)
    ref = orc.decode(enc.packed, enc.norms, 4, 128, 42, out_dtype="f16")
    P.assert_reconstruction_close(host_f64(out), ref, np.linalg.norm(x.astype(np.float64), axis=1))


def test_pr1_workload_full_size():
    """Workload 1 at full size: 4096 fp32 vectors, b = 2; parity and the reported MSE."""
    w = W.pr1()
    x = w.flat()
    enc, codes, norms = check_encode(x, "f32", 2, what="pr1")
    out = B.rrq_decode(torch.from_numpy(codes).to(DEV), torch.from_numpy(norms).to(DEV), 128, 2, 42,
                       out_dtype=torch.float32)
    xh = host_f64(out)
    x64 = x.astype(np.float64)
    nmse = np.mean(np.sum((xh - x64) ** 2, 1) / np.sum(x64 ** 2, 1))
    assert nmse < 1.05 * ocb.distortion(2)


def test_custom_asymmetric_codebook_generic_path():
    rng = np.random.default_rng(3)
    for bits in (2, 3, 4):
        cb = np.sort(rng.normal(size=1 << bits)).astype(np.float32) * 1.3
        x = W.gaussian(500, 128, "f16", seed=bits).flat()
        enc, codes, norms = check_encode(x, "f16", bits, codebook=cb, what=f"asym b={bits}")
        out = B.rrq_decode(torch.from_numpy(enc.packed).to(DEV),
                           torch.from_numpy(enc.norms).to(DEV), 128, bits, 42, codebook=cb,
                           out_dtype=torch.float32)
        ref = orc.decode_exact(enc.packed, enc.norms, bits, 128, 42, levels=cb.astype(np.float64))
        P.assert_rotated_close(host_f64(out), ref, np.linalg.norm(x.astype(np.float64), axis=1))


def test_symmetric_custom_codebook_fast_path():
    cb = (np.arange(16, dtype=np.float32) - 7.5) * np.float32(0.3)  # exactly symmetric
    x = W.gaussian(400, 128, "bf16", seed=9).flat()
    check_encode(x, "bf16", 4, codebook=cb, what="uniform symmetric")


def test_close_thresholds_take_the_compare_search():
    """Two thresholds 0.0005 apart cannot share the cell table; the encoder falls back."""
    cb = np.array([-1.0, 0.0, 0.001, 1.0], dtype=np.float32)
    x = W.gaussian(600, 128, "f16", seed=21).flat()
    check_encode(x, "f16", 2, codebook=cb, what="close thresholds")


@pytest.mark.parametrize("scale", [40.0, 1e-3])
def test_wide_and_narrow_codebooks(scale):
    """Thresholds far outside [−1, 1] (and far inside) move the cell table's range R."""
    cb = (ocb.lloyd_max(4) * scale).astype(np.float32)
    x = W.gaussian(700, 128, "bf16", seed=22).flat()
    check_encode(x, "bf16", 4, codebook=cb, what=f"codebook x{scale}")


@pytest.mark.parametrize("dtype,d,bits", [("f16", 128, 4), ("bf16", 128, 3), ("f16", 64, 2),
                                          ("bf16", 64, 1)])
def test_batch_encoder_several_rounds(dtype, d, bits):
    """Enough batches that every warp of a full grid takes three or more (stage and tile
    reuse, mbarrier phases), plus a ragged last batch; every row against the oracle."""
    n = 148 * 8 * 32 * 3 + 19
    x = W.gaussian(n, d, dtype, seed=23 + bits, scale=1.7).flat()
    check_encode(x, dtype, bits, what=f"rounds {dtype} d={d} b={bits}")


@pytest.mark.parametrize("out_dtype,d", [("f16", 128), ("bf16", 128), ("f32", 128), ("f16", 64)])
def test_batch_decoder_several_rounds(out_dtype, d):
    """4-bit decode over enough batches that every warp of a full grid takes several
    (ring stages, tile reuse, tensor-store clipping of the ragged last batch)."""
    n = 148 * 10 * 32 * 2 + 13
    x = W.gaussian(n, d, "f32", seed=31 + d, scale=1.3).flat().astype(np.float64)
    enc = orc.encode(x, 4, 42)
    out = B.rrq_decode(torch.from_numpy(enc.packed).to(DEV), torch.from_numpy(enc.norms).to(DEV), d, 4,
                       42, out_dtype=TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    ref = orc.decode(enc.packed, enc.norms, 4, d, 42, out_dtype=out_dtype)
    P.assert_reconstruction_close(host_f64(out), ref, np.linalg.norm(x, axis=1),
                                  f"rounds decode {out_dtype} d={d}")


def test_edge_cases_zero_ties_extremes():
    d = 128
    x = np.zeros((9, d), dtype=np.float16)
    x[1, 0] = x[1, 1] = 1.0                 # e1 + e2: exact zeros after the rotation
    x[2, :] = 1.0                           # constant vector
    x[3, 5] = 65504.0                       # fp16 max, one-hot
    x[4, :] = np.float16(6e-8)              # fp16 subnormals
    x[5, ::2] = -65504.0
    x[6, 7] = -1.0
    x[7] = np.float16(-3.0)
    x[8, :64] = 2.0
    for bits in (1, 2, 3, 4):
        enc, codes, norms = check_encode(x, "f16", bits, what=f"edge b={bits}")
        assert norms[0] == 0 and np.all(P.unpack_codes(codes, bits, d)[0] == (1 << (bits - 1)) - 1)
        out = B.rrq_decode(torch.from_numpy(codes).to(DEV), torch.from_numpy(norms).to(DEV), d, bits,
                           42, out_dtype=torch.float32)
        assert torch.all(out[0] == 0)


@pytest.mark.parametrize("n", [0, 1, 2, 15, 17, 255, 257])
def test_small_and_ragged_sizes(n):
    x = W.gaussian(max(n, 1), 128, "f16", seed=n).flat()[:n]
    if n == 0:
        xd = torch.empty(0, 128, dtype=torch.float16, device=DEV)
        codes, norms = B.rrq_encode(xd, 4, 42)
        assert codes.numel() == 0
        return
    check_encode(x, "f16", 4, what=f"n={n}")


def test_full_size_kv_sampled_parity():
    """The benchmarked launch: 262,144 fp16 vectors at b = 4; sampled rows vs the oracle."""
    w = W.kv()
    x = w.flat()
    xd = to_dev(x, "f16")
    codes, norms = B.rrq_encode(xd, 4, 42)
    out = B.rrq_decode(codes, norms, 128, 4, 42, out_dtype=torch.float16)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(0).choice(x.shape[0], 3000, replace=False))
    rows = np.concatenate([rows, [0, x.shape[0] - 1]])
    xs = x[rows].astype(np.float64)
    enc = orc.encode(xs, 4, 42)
    tau = ocb.thresholds(ocb.lloyd_max(4))
    gc = P.unpack_codes(codes[rows].cpu().numpy(), 4, 128)
    P.assert_codes_match(gc, enc.codes, enc.u, tau, "full kv")
    P.assert_norms_close(norms[rows].cpu().numpy(), enc.norm64, 128, "full kv")
    ref = orc.decode(codes[rows].cpu().numpy(), norms[rows].cpu().numpy(), 4, 128, 42, out_dtype="f16")
    P.assert_reconstruction_close(host_f64(out[rows]), ref, np.linalg.norm(xs, axis=1), "full kv")
    # whole-array property: round-trip NMSE of the rotated scheme ≤ the Gaussian D_4 (+5 %)
    xf = xd.float()
    nmse = ((out.float() - xf).pow(2).sum(1) / xf.pow(2).sum(1)).mean().item()
    assert nmse < 1.05 * ocb.distortion(4)


def test_invalid_arguments_raise_without_launch():
    x = torch.zeros(4, 100, dtype=torch.float16, device=DEV)
    with pytest.raises(B.RRQError) as e:
        B.rrq_encode(x, 4, 42)
    assert e.value.status == B.RRQ_ERR_INVALID
    x = torch.zeros(4, 128, dtype=torch.float16, device=DEV)
    with pytest.raises(B.RRQError):
        B.rrq_encode(x, 4, 42, codebook=np.zeros(16, np.float32))
    misaligned = torch.zeros(4 * 128 + 1, dtype=torch.float16, device=DEV)[1:].view(4, 128)
    with pytest.raises(B.RRQError):
        B.rrq_encode(misaligned, 4, 42)
