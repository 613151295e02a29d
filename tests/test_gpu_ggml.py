"""GPU-vs-oracle parity for rrq_ggml_rot / rrq_ggml_rot_decode with the q4_1, q5_0,
q5_1 and q8_0 block types (needs a B200).

Without rotation the GPU takes the same fp32 decisions on the same fp32 values
as the oracle, so the blocks must be equal byte for byte.  With rotation the
GPU's rotated values differ from the oracle's fp32-rounded exact ones by a few
ulps, so:
* a code may differ by one step where the oracle's exact decision quantity lies
  within 1e-5 (in code units) of its rounding boundary; such codes must be
  fewer than 1e-4 of all codes;
* a stored fp16 scalar (scale or min) may differ by one fp16 step where the
  oracle's fp32 scalar lies within 1e-5 (relative) of the fp16 rounding midpoint;
* q5_0 takes its scale from the element of largest |y|: where two elements are
  within 1e-5 (relative) of each other the GPU may pick the other, and the block
  must then be the oracle's encoding for that pick (rare);
* a block of zeros may carry either sign of zero in its scalars.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import ggml_blocks as og
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}
FORMATS = og.FORMATS


def to_dev(x, dtype):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype == "bf16":
        t = t.to(torch.float32).to(torch.bfloat16)
    return t.to(DEV)


def gpu_encode(x, dtype, seed, fmt, rotate):
    out = B.rrq_ggml_rot(to_dev(x, dtype), seed, fmt, rotate=rotate)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _fp16_boundary(v32: float, a: float, b: float) -> bool:
    """fp16 values a != b (same sign) on either side of the fp32 value v32's rounding midpoint."""
    if a == b or np.signbit(a) != np.signbit(b):
        return False
    mid = 0.5 * (a + b)
    return abs(v32 - mid) <= 1e-5 * abs(v32)


def compare_blocks(gpu_blocks, x64, seed, fmt, rotate, what=""):
    n, d = x64.shape
    nb = d // 32
    by = og.BLOCK_BYTES[fmt]
    enc = og.encode(x64, seed, fmt, rotate_first=rotate)
    g = np.asarray(gpu_blocks, np.uint8).reshape(n, nb, by)
    o = enc.blocks.reshape(n, nb, by)
    if not rotate:
        bad = np.argwhere(np.any(g != o, axis=2))
        assert bad.size == 0, f"{what}: {len(bad)} blocks differ without rotation, first {bad[:3].tolist()}"
        return 0, 0
    gs, gm, gq = og.parse_blocks(g.reshape(n, -1), d, fmt)
    os_, om, oq = og.parse_blocks(o.reshape(n, -1), d, fmt)
    gq, oq = gq.reshape(n, nb, 32), oq.reshape(n, nb, 32)
    margin = enc.margin.reshape(n, nb, 32)
    yb = enc.y.reshape(n, nb, 32)
    exempt = ties = 0
    for i, j in np.argwhere(np.any(g != o, axis=2)):
        y = yb[i, j].astype(np.float32)
        if not np.any(y != 0):  # a block of zeros: only the signs of zero may differ
            assert np.all(gq[i, j] == oq[i, j]) and gs[i, j] == os_[i, j] == 0, f"{what}: zero block ({i},{j})"
            continue
        want_q, marg = oq[i, j], margin[i, j]
        if gs[i, j] != os_[i, j]:
            if _fp16_boundary(float(enc.scale32[i, j]), gs[i, j], os_[i, j]):
                exempt += 1
            else:
                assert fmt == "q5_0", f"{what}: block ({i},{j}) scale {gs[i, j]} vs {os_[i, j]}"
                amax = np.abs(y).max()
                cand = [k for k in range(32) if abs(abs(y[k]) - amax) <= 1e-5 * amax
                        and np.float16(np.float32(y[k]) / np.float32(-16.0)) == np.float16(gs[i, j])]
                assert cand, f"{what}: block ({i},{j}) scale {gs[i, j]} vs {os_[i, j]} is not a near-tie"
                ties += 1
                q2, _, _, m2 = og.block_decisions(y[None], fmt, pick=np.array([cand[0]]))
                want_q, marg = q2[0], m2[0]
        if gm[i, j] != om[i, j]:
            assert _fp16_boundary(float(enc.min32[i, j]), gm[i, j], om[i, j]), \
                f"{what}: block ({i},{j}) min {gm[i, j]} vs {om[i, j]}"
            exempt += 1
        diff = gq[i, j] != want_q
        ok = ~diff | ((np.abs(gq[i, j] - want_q) == 1) & (marg < 1e-5))
        assert np.all(ok), f"{what}: block ({i},{j}) codes differ outside the band"
        exempt += int(np.sum(diff))
    assert exempt < 1e-4 * n * d + 2, f"{what}: {exempt} exempt codes / scalars of {n * d}"
    assert ties <= max(2, 1e-3 * n * nb), f"{what}: {ties} near-tie blocks"
    return exempt, ties


def test_hand_worked_golden_blocks_on_gpu():
    from tests.test_oracle_pins import _ggml_inputs, _golden_lines
    rows = {}
    for ln in _golden_lines("ggml_blocks.txt"):
        fmt, name, hexbytes = (p.strip() for p in ln.split("|"))
        rows.setdefault(fmt, []).append((name, bytes.fromhex(hexbytes.replace(" ", ""))))
    for fmt, items in rows.items():
        nblk = 2
        while nblk < len(items):
            nblk *= 2
        x = np.zeros((1, 32 * max(nblk, 2)), np.float32)
        for k, (name, _) in enumerate(items):
            x[0, 32 * k:32 * (k + 1)] = _ggml_inputs(name)
        got = gpu_encode(x, "f32", 0, fmt, rotate=False).reshape(-1, og.BLOCK_BYTES[fmt])
        for k, (name, want) in enumerate(items):
            assert bytes(got[k]) == want, (fmt, name, bytes(got[k]).hex())


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("rotate", [False, True])
def test_ggml_encode_parity(fmt, dtype, d, rotate):
    # several grid-stride passes of the 64-block warp tiles plus a ragged tail
    x = W.gaussian(1111, d, dtype, seed=d + 3 * len(fmt) + (5 if rotate else 0), scale=2.0).flat()
    out = gpu_encode(x, dtype, 42, fmt, rotate)
    compare_blocks(out, x.astype(np.float64), 42, fmt, rotate, f"{fmt} {dtype} d={d} rot={rotate}")


@pytest.mark.parametrize("fmt", FORMATS)
@pytest.mark.parametrize("out_dtype", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128, 512])
@pytest.mark.parametrize("rotate", [False, True])
def test_ggml_decode_parity_on_oracle_blocks(fmt, out_dtype, d, rotate):
    x = W.gaussian(301, d, "f32", seed=d + 11, scale=1.5).flat().astype(np.float64)
    enc = og.encode(x, 42, fmt, rotate_first=rotate)
    out = B.rrq_ggml_rot_decode(torch.from_numpy(enc.blocks).to(DEV), d, 42, fmt, rotate=rotate,
                                out_dtype=TORCH_DT[out_dtype])
    torch.cuda.synchronize()
    got = out.to(torch.float64).cpu().numpy()
    xn = np.linalg.norm(x, axis=1)
    ref = og.decode(enc.blocks, d, 42, fmt, rotate_first=rotate, out_dtype=out_dtype)
    P.assert_reconstruction_close(got, ref, xn, f"{fmt} decode {out_dtype} d={d} rot={rotate}")
    if out_dtype == "f32":
        exact = og.decode_exact(enc.blocks, d, 42, fmt, rotate_first=rotate)
        P.assert_rotated_close(got, exact, xn, f"{fmt} decode f32 tight")


@pytest.mark.parametrize("fmt", FORMATS)
def test_ggml_zero_rows_ragged_sizes_and_round_trip(fmt):
    x = W.gaussian(70, 128, "f16", seed=9, scale=3.0).flat().copy()
    x[[0, 33, 69]] = 0
    for n in (1, 17, 33, 70):
        out = gpu_encode(x[:n], "f16", 42, fmt, True)
        compare_blocks(out, x[:n].astype(np.float64), 42, fmt, True, f"{fmt} n={n}")
    blk = B.rrq_ggml_rot(to_dev(x, "f16"), 42, fmt)
    back = B.rrq_ggml_rot_decode(blk, 128, 42, fmt, out_dtype=torch.float32)
    torch.cuda.synchronize()
    back = back.cpu().numpy()
    assert np.all(back[[0, 33, 69]] == 0)
    # the round trip error matches the oracle's own round trip
    x64 = x.astype(np.float64)
    ref = og.decode_exact(og.encode(x64, 42, fmt).blocks, 128, 42, fmt)
    err = np.linalg.norm(back - x64, axis=1)
    err_ref = np.linalg.norm(ref - x64, axis=1)
    assert np.all(np.abs(err - err_ref) <= 2e-3 * np.linalg.norm(x64, axis=1)), fmt
    e = B.rrq_ggml_rot(torch.empty(0, 128, dtype=torch.float16, device=DEV), 42, fmt)
    assert e.shape == (0, 4 * og.BLOCK_BYTES[fmt])


@pytest.mark.parametrize("fmt", FORMATS)
def test_ggml_full_size_sampled_and_rotation_gain(fmt):
    """The Attn-rot workload shape (131072 tokens x 8 heads x 128, fp16, outlier channels):
    sampled parity at full size, and the rotated error below the unrotated one."""
    w = W.attnrot()
    x = w.flat()
    xd = to_dev(x, "f16")
    out = B.rrq_ggml_rot(xd, 42, fmt).cpu().numpy()
    rows = np.random.default_rng(3).choice(x.shape[0], 1500, replace=False)
    rows.sort()
    compare_blocks(out[rows], x[rows].astype(np.float64), 42, fmt, True, f"{fmt} full-size sample")
    mse = {}
    for rot in (True, False):
        blk = B.rrq_ggml_rot(xd, 42, fmt, rotate=rot)
        back = B.rrq_ggml_rot_decode(blk, 128, 42, fmt, rotate=rot, out_dtype=torch.float32)
        mse[rot] = float(torch.mean((back - xd.float()) ** 2))
    assert mse[True] < mse[False], (fmt, mse)


def test_q4_0_through_the_block_type_entry_and_signed_zero_blocks():
    """rrq_ggml_rot(q4_0) writes what rrq_q4_0_rot writes, and its decode matches;
    blocks of −0 store the −0 scale (GGML starts its signed max at +0)."""
    from oracle import q4_0 as oq
    x = W.gaussian(257, 256, "bf16", seed=77, scale=1.3).flat().copy()
    x[5] = -0.0
    xd = to_dev(x, "bf16")
    a = B.rrq_ggml_rot(xd, 42, "q4_0", rotate=False)
    b = B.rrq_q4_0_rot(xd, 42, rotate=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    enc = oq.encode(x.astype(np.float64), 42, rotate_first=False)
    assert np.array_equal(a.cpu().numpy(), enc.blocks)
    assert a[5].cpu().numpy().reshape(8, 18)[:, :2].tobytes() == b"\x00\x80" * 8
    da = B.rrq_ggml_rot_decode(a, 256, 42, "q4_0", rotate=False, out_dtype=torch.float32)
    db = B.rrq_q4_0_rot_decode(b, 256, 42, rotate=False, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(da, db)
