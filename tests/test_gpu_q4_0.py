"""GPU-vs-oracle parity for rrq_q4_0_rot / rrq_q4_0_rot_decode (needs a B200).

Codes decided in floating point: a code may differ from the oracle's only when
the oracle's y/Δ + 8.5 lies within 1e-5 of an integer.  The block scale is an
argmax; when two elements of a block have |y| within 1e-5 (relative) of each
other, fp32 may pick the other one: such a block must then be exactly the
oracle's encoding for the GPU's choice, and such blocks must be rare.
"""

from __future__ import annotations

import os

import numpy as np
import pytest
import torch

from oracle import q4_0 as oq
from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q4_0_blocks.txt")


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)
    return t.to(DEV)


def compare_blocks(gpu_blocks, x64, seed, rotate, what=""):
    """Returns the number of exempt codes and near-tie blocks; asserts the rest is exact."""
    n, d = x64.shape
    nb = d // 32
    enc = oq.encode(x64, seed, rotate_first=rotate)
    g = np.asarray(gpu_blocks, np.uint8).reshape(n, nb, 18)
    o = enc.blocks.reshape(n, nb, 18)
    yb = enc.y.reshape(n, nb, 32)
    exempt = ties = 0
    for i, j in zip(*np.nonzero(np.any(g != o, axis=2))):
        gd = g[i, j, :2].view(np.float16)[0]
        od = o[i, j, :2].view(np.float16)[0]
        y = yb[i, j]
        od32 = float(enc.delta[i, j])
        mid = 0.5 * (float(gd) + float(od))
        scale_boundary = (np.signbit(gd) == np.signbit(od) and gd != od
                          and abs(od32 - mid) <= 1e-5 * abs(od32))
        if (gd != od or np.signbit(gd) != np.signbit(od)) and not scale_boundary:
            # near-tie: the GPU's scale must come from an element within 1e-5 of the max |y|
            cand = [k for k in range(32) if abs(abs(y[k]) - np.abs(y).max()) <= 1e-5 * np.abs(y).max()
                    and abs(float(np.float16(np.float32(y[k]) / np.float32(-8.0))) - float(gd))
                    <= 2 * abs(float(np.spacing(np.float16(gd))))]
            assert cand, f"{what}: block ({i},{j}) scale {gd} vs {od} is not a near-tie"
            ties += 1
            # the oracle's fp32 decision rule, with the GPU's choice of scale element
            delta = np.float32(np.float32(y[cand[0]]) / np.float32(-8.0))
            inv = np.float32(1.0) / delta if delta != 0 else np.float32(0.0)
            r32 = (y.astype(np.float32) * inv).astype(np.float32) + np.float32(8.5)
            want = np.minimum(15, np.maximum(0, np.floor(r32))).astype(np.int64)
            ratio = y * float(inv) + 8.5
        else:
            # same element; a stored scale may differ by one fp16 step when the fp32
            # scale lies on an fp16 rounding boundary (codes use the fp32 scale)
            exempt += int(scale_boundary)
            ratio = enc.ratio.reshape(n, nb, 32)[i, j]
            want = enc.q.reshape(n, nb, 32)[i, j]
        got = np.concatenate([g[i, j, 2:] & 15, g[i, j, 2:] >> 4]).astype(np.int64)
        bad = got != want
        near = np.abs(ratio - np.round(ratio)) < 1e-5
        assert not np.any(bad & ~near), f"{what}: block ({i},{j}) codes differ outside the band"
        exempt += int(np.sum(bad))
    total = n * d
    assert exempt < 1e-4 * total + 1, f"{what}: {exempt} exempt codes of {total}"
    assert ties <= max(2, 1e-3 * n * nb), f"{what}: {ties} near-tie blocks"
    return exempt, ties


def test_hand_worked_golden_blocks_on_gpu():
    from tests.test_oracle_pins import _golden_lines, _q4_inputs
    names, want = [], []
    for ln in _golden_lines("q4_0_blocks.txt"):
        name, _, hexbytes = (p.strip() for p in ln.split("|"))
        names.append(name)
        want.append(bytes.fromhex(hexbytes.replace(" ", "")))
    # two blocks per vector (d = 64): pair the six hand-worked blocks into three vectors
    x = np.stack([np.concatenate([_q4_inputs(names[2 * i]), _q4_inputs(names[2 * i + 1])])
                  for i in range(3)]).astype(np.float32)
    out = B.rrq_q4_0_rot(to_dev(x, "f32"), 0, rotate=False)
    torch.cuda.synchronize()
    got = out.cpu().numpy().reshape(6, 18)
    for k in range(6):
        assert bytes(got[k]) == want[k], names[k]


@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("rotate", [True, False])
def test_q4_0_encode_parity(dtype, d, rotate):
    x = W.gaussian(333, d, dtype, seed=d + (7 if rotate else 0), scale=2.0).flat()
    out = B.rrq_q4_0_rot(to_dev(x, dtype), 42, rotate=rotate)
    torch.cuda.synchronize()
    compare_blocks(out.cpu().numpy(), x.astype(np.float64), 42, rotate, f"q4_0 {dtype} d={d} rot={rotate}")


@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("rotate", [True, False])
def test_q4_0_decode_parity_on_oracle_blocks(out_dtype, d, rotate):
    x = W.gaussian(301, d, "f32", seed=d + 11, scale=1.5).flat().astype(np.float64)
    enc = oq.encode(x, 42, rotate_first=rotate)
    out = B.rrq_q4_0_rot_decode(torch.from_numpy(enc.blocks).to(DEV), d, 42, rotate=rotate,
                                out_dtype=TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    ref = oq.decode(enc.blocks, d, 42, rotate_first=rotate, out_dtype=out_dtype)
    xn = np.linalg.norm(x, axis=1)
    got = out.to(torch.float64).cpu().numpy()
    P.assert_reconstruction_close(got, ref, xn, f"q4 decode {out_dtype} d={d} rot={rotate}")
    if out_dtype == "f32":
        exact = oq.decode_exact(enc.blocks, d, 42, rotate_first=rotate)
        P.assert_rotated_close(got, exact, xn, "q4 decode f32 tight")


@pytest.mark.parametrize("n", [1, 3, 17, 33, 255])
def test_q4_0_ragged_sizes(n):
    x = W.gaussian(n, 128, "f16", seed=n).flat()
    out = B.rrq_q4_0_rot(to_dev(x, "f16"), 42)
    dec = B.rrq_q4_0_rot_decode(out, 128, 42)
    torch.cuda.synchronize()
    compare_blocks(out.cpu().numpy(), x.astype(np.float64), 42, True, f"n={n}")
    assert dec.shape == (n, 128)


def test_q4_0_full_size_sampled_and_rotation_gain():
    """Workload 3: 1M fp16 KV vectors; sampled parity and the MSE ratio rotated/unrotated."""
    w = W.attnrot()
    x = w.flat()
    xd = to_dev(x, "f16")
    rows = np.sort(np.random.default_rng(2).choice(x.shape[0], 2000, replace=False))
    mse = {}
    for rot in (True, False):
        blk = B.rrq_q4_0_rot(xd, 42, rotate=rot)
        dec = B.rrq_q4_0_rot_decode(blk, 128, 42, rotate=rot, out_dtype=torch.float32)
        torch.cuda.synchronize()
        compare_blocks(blk[torch.from_numpy(rows).to(DEV)].cpu().numpy(), x[rows].astype(np.float64),
                       42, rot, f"full rot={rot}")
        xf = xd.float()
        mse[rot] = ((dec - xf) ** 2).mean().item()
    assert mse[True] < mse[False]
