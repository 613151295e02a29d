"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test pins one oracle function to something other than itself: a value the
pages print, a published table or test vector, a closed form, an invariant, a
library routine, or brute force on tiny inputs.
"""

from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.stats

from oracle import attention, codebook, ggml_blocks, hadamard, q4_0, qjl, rng, rrq, sphere

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


# --------------------------------------------------------------------------- rng
def test_splitmix64_published_vector():
    for ln in _golden_lines("splitmix64_vectors.txt"):
        seed, idx, out = (int(v) for v in ln.split())
        assert rng.splitmix64(seed, 1, start=idx)[0] == out


def test_rotation_signs_balanced_and_deterministic():
    s = rng.rotation_signs(42, 4096)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 4 / math.sqrt(4096)
    assert np.array_equal(s, rng.rotation_signs(42, 4096))
    # prefix property: the sign of coordinate i does not depend on d
    assert np.array_equal(rng.rotation_signs(42, 64), s[:64])
    assert not np.array_equal(rng.rotation_signs(43, 64), s[:64])


def test_bf16_round_ties_and_no_double_rounding():
    # exactly halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert rng.bf16_round(np.array([1 + 2.0 ** -8]))[0] == 1.0
    # halfway between 1 + 2^-7 and 1 + 2^-6: ties to even -> 1 + 2^-6
    assert rng.bf16_round(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    # just above the tie must round up; a float32 intermediate would lose the 2^-40
    assert rng.bf16_round(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1 + 2.0 ** -7
    assert rng.bf16_round(np.array([-3.0]))[0] == -3.0
    assert rng.bf16_round(np.array([0.0]))[0] == 0.0


def test_f16_output_rounding_single_step():
    # same double-rounding trap for fp16 outputs
    v = np.array([1 + 2.0 ** -11 + 2.0 ** -40, 1 + 2.0 ** -11])
    out = rrq.round_to(v, "f16")
    assert out[0] == 1 + 2.0 ** -10 and out[1] == 1.0


def test_qjl_gaussian_moments_and_bf16_exact():
    s = rng.qjl_gaussian(4242, 64)
    assert np.array_equal(s, rng.bf16_round(s))
    flat = s.ravel()
    assert abs(flat.mean()) < 5 / math.sqrt(flat.size)
    assert abs(flat.var() - 1.0) < 0.05
    # a normal sample: kurtosis ~3, symmetric
    assert abs(scipy.stats.kurtosis(flat, fisher=False) - 3.0) < 0.3
    assert scipy.stats.kstest(flat, "norm").pvalue > 1e-3


# --------------------------------------------------------------------- hadamard
@pytest.mark.parametrize("d", [1, 2, 4, 8, 64, 128, 256, 512])
def test_sylvester_orthogonal_and_matches_scipy(d):
    h = hadamard.sylvester(d)
    assert np.array_equal(h @ h.T, d * np.eye(d))
    assert np.array_equal(h, scipy.linalg.hadamard(d).astype(np.float64))


def test_sylvester_entry_closed_form_d8():
    # H_ij = (-1)^popcount(i & j) for Sylvester's natural order
    d = 8
    ref = np.array([[(-1) ** bin(i & j).count("1") for j in range(d)] for i in range(d)], dtype=float)
    assert np.array_equal(hadamard.sylvester(d), ref)


@pytest.mark.parametrize("d", [64, 128, 512])
def test_rotation_is_orthogonal_and_signs_first(d):
    p = hadamard.rotation_matrix(42, d)
    assert np.allclose(p @ p.T, np.eye(d), atol=1e-12)
    x = np.random.default_rng(0).standard_normal((5, d))
    assert np.allclose(np.linalg.norm(rrq.rotate(x, 42), axis=1), np.linalg.norm(x, axis=1))
    # Π = H·D/√d: (H/√d)ᵀ Π must be diagonal with ±1 entries (signs applied first)
    dmat = (hadamard.sylvester(d) / math.sqrt(d)).T @ p
    assert np.allclose(dmat, np.diag(np.diag(dmat)), atol=1e-12)
    assert np.allclose(np.abs(np.diag(dmat)), 1.0)
    # inverse really inverts
    assert np.allclose(rrq.rotate(rrq.rotate(x, 42), 42, inverse=True), x, atol=1e-12)


@pytest.mark.parametrize("d", [8, 16])
def test_sign_enumeration_moments_exact(d):
    """Over all 2^d sign vectors D: E[(H D x/√d)_i] = 0 and E[(H D x/√d)_i²] = ‖x‖²/d exactly."""
    x = np.random.default_rng(d).standard_normal(d)
    h = hadamard.sylvester(d) / math.sqrt(d)
    signs = np.array(list(itertools.product([-1.0, 1.0], repeat=d)))  # [2^d, d]
    y = (signs * x[None, :]) @ h.T  # rows: H·D·x/√d
    assert np.allclose(y.mean(axis=0), 0.0, atol=1e-12)
    assert np.allclose((y ** 2).mean(axis=0), np.dot(x, x) / d, rtol=1e-12)


# ----------------------------------------------------------------------- sphere
@pytest.mark.parametrize("d", [3, 8, 16, 128])
def test_marginal_density_normalised(d):
    from scipy.integrate import quad
    total, _ = quad(lambda t: sphere.marginal_density(np.array([t]), d)[0], -1, 1, limit=200)
    assert abs(total - 1.0) < 1e-9


def test_marginal_density_special_cases():
    xs = np.linspace(-0.99, 0.99, 11)
    assert np.allclose(sphere.marginal_density(xs, 3), 0.5)  # d=3: uniform on [-1, 1]
    for d in (8, 128):
        a = (d - 1) / 2.0
        ref = scipy.stats.beta.pdf((xs + 1) / 2, a, a) / 2
        assert np.allclose(sphere.marginal_density(xs, d), ref, rtol=1e-10)


def test_marginal_std_page_value_d1000():
    # "at d = 1000 the standard deviation is about 0.032"
    from scipy.integrate import quad
    d = 1000
    var, _ = quad(lambda t: t * t * sphere.marginal_density(np.array([t]), d)[0], -1, 1, points=[0], limit=400)
    assert abs(math.sqrt(var) - 1 / math.sqrt(d)) < 1e-9
    assert round(math.sqrt(var), 3) == 0.032


@pytest.mark.parametrize("d", [64, 128])
def test_rotated_gaussian_matches_sphere_marginal(d):
    """Πx/‖x‖ for Gaussian x is uniform on the sphere: mean 0, std 1/√d, Beta marginal (KS)."""
    g = np.random.default_rng(100 + d).standard_normal((4000, d))
    y = rrq.rotate(g, 42)
    z = y / np.linalg.norm(y, axis=1, keepdims=True)
    col = z[:, 5]
    assert abs(col.mean()) < 4 / math.sqrt(d * 4000)
    assert abs(z.std() - 1 / math.sqrt(d)) < 0.01 / math.sqrt(d)
    a = (d - 1) / 2.0
    assert scipy.stats.kstest((col + 1) / 2, lambda t: scipy.stats.beta.cdf(t, a, a)).pvalue > 1e-3


def test_marginal_tends_to_normal():
    gaps = []
    for d in (8, 32, 128, 512):
        xs = np.linspace(-1, 1, 20001)
        f = sphere.marginal_density(xs, d)
        cdf = np.cumsum(f) * (xs[1] - xs[0])
        gaps.append(np.max(np.abs(cdf - scipy.stats.norm.cdf(xs * math.sqrt(d)))))
    assert all(a > b for a, b in zip(gaps, gaps[1:]))
    assert gaps[-1] < 2e-3


# --------------------------------------------------------------------- codebook
def test_codebook_one_bit_closed_form():
    c = codebook.lloyd_max(1)
    assert abs(c[1] - math.sqrt(2 / math.pi)) < 1e-12 and abs(c[0] + c[1]) < 1e-15
    assert abs(codebook.distortion(1) - (1 - 2 / math.pi)) < 1e-12


def test_codebook_page_values():
    for ln in _golden_lines("codebook_page.txt"):
        parts = ln.split()
        bits, vals = int(parts[0]), [float(v) for v in parts[1:]]
        c = codebook.lloyd_max(bits)
        pos = c[len(c) // 2:]
        assert [round(v, 3) for v in pos] == vals


def test_codebook_max1960_table():
    for ln in _golden_lines("codebook_max1960.txt"):
        parts = ln.split()
        bits, kind, vals = int(parts[0]), parts[1], [float(v) for v in parts[2:]]
        c = codebook.lloyd_max(bits)
        if kind == "levels":
            assert np.allclose(c[len(c) // 2:], vals, atol=2e-4, rtol=5e-4)
        elif kind == "thresholds":
            t = codebook.thresholds(c)
            assert np.allclose(t[len(t) // 2 + 1:], vals, atol=2e-4, rtol=5e-4)
        else:
            assert abs(codebook.distortion(bits) - vals[0]) < 1e-3 * vals[0]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_codebook_fixed_point_symmetry_and_distortion(bits):
    c = codebook.lloyd_max(bits)
    assert np.all(np.diff(c) > 0)
    assert np.allclose(c, -c[::-1], atol=1e-13)
    assert np.max(np.abs(codebook.lloyd_step(c) - c)) < 1e-12
    # two independent distortion formulas agree
    assert abs(codebook.quantize_distortion(c) - codebook.distortion(bits)) < 1e-12
    # Monte Carlo distortion of nearest-level quantisation
    g = np.random.default_rng(bits).standard_normal(400000)
    qv = c[np.argmin(np.abs(g[:, None] - c[None, :]), axis=1)]
    mc = np.mean((g - qv) ** 2)
    assert abs(mc - codebook.distortion(bits)) < 5 * np.std((g - qv) ** 2) / math.sqrt(g.size)


def test_codebook_distortion_decreases_with_bits():
    ds = [codebook.distortion(b) for b in range(1, 6)]
    assert all(a > b for a, b in zip(ds, ds[1:]))


# --------------------------------------------------------------- encode / decode
def _nearest_codes(u, levels):
    """Brute force: index of the nearest centroid; ties (equal distance) to the lower one."""
    dist = np.abs(u[..., None] - levels)
    return np.argmin(dist, axis=-1)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [8, 64, 128])
def test_codes_are_nearest_centroid(bits, d):
    x = np.random.default_rng(bits * 100 + d).standard_normal((300, d)) * 3
    enc = rrq.encode(x, bits, 42)
    c = codebook.lloyd_max(bits)
    assert np.array_equal(enc.codes, _nearest_codes(enc.u, c))
    # u really is sqrt(d)·Πx/‖x‖ with the orthogonal Π
    assert np.allclose(np.linalg.norm(enc.u, axis=1), math.sqrt(d))


def _pack_bitwise(codes, bits):
    out = []
    for row in codes:
        stream = []
        for v in row:
            stream.extend((int(v) >> k) & 1 for k in range(bits))
        out.append([sum(stream[8 * j + k] << k for k in range(8)) for j in range(len(stream) // 8)])
    return np.array(out, dtype=np.uint8)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_matches_bitwise_reference(bits):
    codes = np.random.default_rng(bits).integers(0, 1 << bits, size=(7, 64))
    packed = rrq.pack_codes(codes, bits)
    assert np.array_equal(packed, _pack_bitwise(codes, bits))
    assert np.array_equal(rrq.unpack_codes(packed, bits, 64), codes)
    if bits == 4:  # coordinate 2j in the low nibble of byte j
        assert packed[0, 0] == (codes[0, 0] | (codes[0, 1] << 4))


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_round_trip_nmse_matches_lloyd_max_distortion(bits):
    d, n = 128, 3000
    x = np.random.default_rng(7 + bits).standard_normal((n, d))
    enc = rrq.encode(x, bits, 42)
    xh = rrq.decode_exact(enc.packed, enc.norms, bits, d, 42)
    err = np.sum((x - xh) ** 2, axis=1) / np.sum(x * x, axis=1)
    # finite-d (Beta) marginal differs slightly from N(0,1): allow 3 % + MC noise
    tol = 0.03 * codebook.distortion(bits) + 5 * err.std() / math.sqrt(n)
    assert abs(err.mean() - codebook.distortion(bits)) < tol


def test_outlier_channels_dissolved_by_rotation():
    """Workload 1: rotated NMSE ≈ D_2 while the unrotated scheme is far worse."""
    from random_rotation_kv_b200 import workloads
    w = workloads.pr1(n=2000)
    x = w.flat().astype(np.float64)
    enc = rrq.encode(x, 2, 42)
    xh = rrq.decode_exact(enc.packed, enc.norms, 2, 128, 42)
    nmse_rot = np.mean(np.sum((x - xh) ** 2, 1) / np.sum(x * x, 1))
    # same codebook, same per-vector scale, no rotation
    c = codebook.lloyd_max(2)
    nu = np.linalg.norm(x, axis=1, keepdims=True)
    u = math.sqrt(128) * x / nu
    xq = c[np.searchsorted(codebook.thresholds(c), u)] * nu / math.sqrt(128)
    nmse_plain = np.mean(np.sum((x - xq) ** 2, 1) / np.sum(x * x, 1))
    # a fixed RHT of a vector dominated by 3 channels gives a clustered (not
    # Gaussian) marginal, so the error can fall below D_2; it must not exceed it
    assert nmse_rot < 1.05 * codebook.distortion(2)
    assert nmse_plain > 3 * nmse_rot


def test_mse_decoder_shrinks_inner_products():
    """"Bias vs unbiasedness": E<x̂, x> = E‖x̂‖² < ‖x‖² for the MSE quantiser."""
    d = 128
    x = np.random.default_rng(3).standard_normal((4000, d))
    enc = rrq.encode(x, 2, 42)
    xh = rrq.decode_exact(enc.packed, enc.norms, 2, d, 42)
    ip = np.sum(xh * x, 1) / np.sum(x * x, 1)
    sq = np.sum(xh * xh, 1) / np.sum(x * x, 1)
    assert ip.mean() < 1 - 0.5 * codebook.distortion(2)
    assert abs(ip.mean() - sq.mean()) < 0.01


def test_zero_vector_and_exact_ties():
    d = 64
    x = np.zeros((3, d))
    x[1, 0] = x[1, 1] = 1.0  # e1 + e2: many exact zeros after the rotation
    enc = rrq.encode(x, 4, 42)
    assert np.all(enc.codes[0] == 7) and enc.norms[0] == 0
    assert np.all(rrq.decode_exact(enc.packed[:1], enc.norms[:1], 4, d, 42) == 0)
    zeros = enc.u[1] == 0
    assert zeros.sum() > 0 and np.all(enc.codes[1][zeros] == 7)
    # exact tie on a non-zero threshold goes to the lower code
    c = codebook.lloyd_max(4)
    tau = codebook.thresholds(c)
    assert np.searchsorted(tau, [tau[10]], side="left")[0] == 10


def test_scores_equal_inner_product_with_reconstruction():
    rg = np.random.default_rng(11)
    t_len, hkv, hq, d, bits = 9, 2, 8, 64, 3
    k = rg.standard_normal((t_len * hkv, d))
    q = rg.standard_normal((hq, d))
    enc = rrq.encode(k, bits, 5)
    s = rrq.scores(q, enc.packed, enc.norms, t_len, hkv, d, bits, 5, scale=0.5)
    xh = rrq.decode_exact(enc.packed, enc.norms, bits, d, 5).reshape(t_len, hkv, d)
    for h in range(hq):
        g = h // (hq // hkv)
        assert np.allclose(s[h], 0.5 * xh[:, g, :] @ q[h], rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------ DRIVE
@pytest.mark.parametrize("d", [8, 16])
def test_drive_biased_scale_is_mse_optimal(d):
    rg = np.random.default_rng(d)
    p = hadamard.rotation_matrix(9, d)
    for _ in range(5):
        x = rg.standard_normal(d) * rg.uniform(0.1, 10)
        rx = p @ x
        s_star = sphere.drive_scale_biased(rx[None])[0]
        grid = np.linspace(0, 3 * s_star, 30001)
        base = sphere.drive_decode(p, x[None], np.array([1.0]))[0]
        errs = [np.sum((x - s * base) ** 2) for s in grid]
        assert abs(grid[int(np.argmin(errs))] - s_star) <= 3 * s_star / 30000


@pytest.mark.parametrize("d", [8, 16])
def test_drive_unbiased_scale(d):
    rg = np.random.default_rng(50 + d)
    x = rg.standard_normal(d)
    p = hadamard.rotation_matrix(3, d)
    rx = p @ x
    s = sphere.drive_scale_unbiased(x[None], rx[None])
    xh = sphere.drive_decode(p, x[None], s)[0]
    assert abs(np.dot(xh, x) - np.dot(x, x)) < 1e-12 * np.dot(x, x)  # per draw
    # unbiased over uniformly random (Haar) rotations: Monte Carlo
    acc = np.zeros(d)
    n = 20000
    for _ in range(n):
        a = rg.standard_normal((d, d))
        qm, r = np.linalg.qr(a)
        qm = qm * np.sign(np.diag(r))[None, :]
        rx = qm @ x
        acc += sphere.drive_decode(qm, x[None], sphere.drive_scale_unbiased(x[None], rx[None]))[0]
    mean = acc / n
    assert np.linalg.norm(mean - x) < 0.05 * np.linalg.norm(x)


@pytest.mark.parametrize("unbiased", [False, True])
def test_drive_encode_through_the_one_bit_decoder(unbiased):
    """drive_encode + the b-bit decoder (codebook {−1, +1}, stored S·√d) is the DRIVE
    mean decoder S·Πᵀ·sign(Πx); the scores path gives S·⟨Πq, sign(Πx)⟩."""
    rg = np.random.default_rng(7)
    x = rg.standard_normal((40, 16)) * rg.uniform(0.5, 3, size=(40, 1))
    enc = sphere.drive_encode(x, 11, unbiased)
    p = hadamard.rotation_matrix(11, 16)
    want = sphere.drive_decode(p, x, enc.scale)
    pm = np.array([-1.0, 1.0])
    got = rrq.decode_exact(enc.packed, enc.stored.astype(np.float64), 1, 16, 11, levels=pm)
    assert np.allclose(got, want, rtol=1e-6, atol=1e-12)
    q = rg.standard_normal((2, 16))
    sc = rrq.scores(q, enc.packed, enc.stored.astype(np.float64), 40, 1, 16, 1, 11, levels=pm)
    want_s = enc.scale[None, :] * ((q @ p.T) @ (2.0 * enc.signs.T - 1.0))
    assert np.allclose(sc, want_s, rtol=1e-6, atol=1e-12)
    if unbiased:
        assert np.allclose(np.sum(got * x, 1), np.sum(x * x, 1), rtol=1e-6)  # <x̂, x> = ‖x‖²


def test_drive_zero_coordinates_take_the_minus_one_sign():
    """A coordinate with (Πx)_i = 0 exactly gets bit 0 (−1) in the encoder and
    in the mean decoder alike.  d = 16 makes Π's entries ±1/4 (exact), so
    x = Πᵀ·(4, 0, …, 0) rotates back to exactly (4, 0, …, 0)."""
    p = hadamard.rotation_matrix(5, 16)
    y = np.zeros(16)
    y[0] = 4.0
    x = (p.T @ y)[None]
    assert np.array_equal(rrq.rotate(x, 5)[0], y)
    for unbiased in (False, True):
        enc = sphere.drive_encode(x, 5, unbiased)
        assert enc.signs[0].tolist() == [1] + [0] * 15
        assert enc.scale[0] == (4.0 / 16 if not unbiased else 16.0 / 4.0)
        want = sphere.drive_decode(p, x, enc.scale)
        got = rrq.decode_exact(enc.packed, enc.stored.astype(np.float64), 1, 16, 5,
                               levels=np.array([-1.0, 1.0]))
        assert np.allclose(got, want, rtol=1e-6, atol=1e-12)
        assert np.allclose(want[0], enc.scale[0] * (p.T @ np.where(y > 0, 1.0, -1.0)))


# ------------------------------------------------------------------------- q4_0
def _q4_inputs(name):
    x = np.zeros(32)
    if name == "ones":
        x[:] = 1.0
    elif name == "outlier":
        x[5] = -4.0
    elif name == "grid":
        x = (((np.arange(32) * 7) % 16) - 8) * 0.25
    elif name == "posmax":
        x[:] = 1.0
        x[0] = 3.0
    elif name == "tie":
        x[2], x[7] = 2.0, -2.0
    return x


def test_q4_0_hand_worked_blocks():
    for ln in _golden_lines("q4_0_blocks.txt"):
        name, _, hexbytes = (p.strip() for p in ln.split("|"))
        want = bytes.fromhex(hexbytes.replace(" ", ""))
        enc = q4_0.encode(_q4_inputs(name)[None], 0, rotate_first=False)
        assert bytes(enc.blocks[0]) == want, name


def test_q4_0_grid_round_trip_exact_and_rotation_equivalence():
    rg = np.random.default_rng(4)
    d = 128
    delta = 2.0 ** rg.integers(-4, 3, size=(6, d // 32))
    k = rg.integers(0, 16, size=(6, d))
    k[:, ::32] = 0  # force the largest magnitude to be -8·Δ (exact grid, valid Δ)
    x = ((k - 8).reshape(6, d // 32, 32) * delta[:, :, None]).reshape(6, d)
    enc = q4_0.encode(x, 0, rotate_first=False)
    assert np.array_equal(enc.q, k)
    assert np.array_equal(q4_0.decode_exact(enc.blocks, d, 0, rotate_first=False), x)
    # rotate=1 is rotate=0 applied to Πx, and decode applies Πᵀ
    y = rg.standard_normal((6, d))
    e1 = q4_0.encode(y, 42, rotate_first=True)
    e0 = q4_0.encode(rrq.rotate(y, 42), 0, rotate_first=False)
    assert np.array_equal(e1.blocks, e0.blocks)
    back = q4_0.decode_exact(e1.blocks, d, 42, rotate_first=True)
    assert np.allclose(rrq.rotate(back, 42), q4_0.decode_exact(e0.blocks, d, 0, rotate_first=False))


def test_q4_0_rotation_lowers_error_on_outlier_inputs():
    from random_rotation_kv_b200 import workloads
    w = workloads.kv(tokens=256)
    x = w.flat().astype(np.float64)
    mse = {}
    for rot in (True, False):
        enc = q4_0.encode(x, 42, rotate_first=rot)
        mse[rot] = np.mean((q4_0.decode_exact(enc.blocks, 128, 42, rotate_first=rot) - x) ** 2)
    assert mse[True] < 0.8 * mse[False]


# -------------------------------------------------------------------------- QJL
def test_qjl_projection_double_loop_tiny():
    d = 8
    rg = np.random.default_rng(1)
    x = rg.standard_normal((3, d))
    s = rng.qjl_gaussian(17, d)
    enc = qjl.encode(x, 2, 42, s)
    for n in range(3):
        for i in range(d):
            v = sum(s[i, j] * enc.r[n, j] for j in range(d))
            assert abs(v - enc.v[n, i]) < 1e-12
            bit = (enc.bits[n, i // 8] >> (i % 8)) & 1
            assert bit == (1 if v > 0 else 0)
        assert abs(enc.rnorm[n] - np.linalg.norm(enc.r[n])) < 1e-6 * np.linalg.norm(enc.r[n])


def test_qjl_estimator_unbiased_monte_carlo():
    """E_S[√(π/2)/m·ρ·<S q', sign(S r)>] = <q', r> over Gaussian S."""
    d = 32
    rg = np.random.default_rng(5)
    x = rg.standard_normal((1, d))
    q = rg.standard_normal(d)
    _, r = qjl.residual(x, 2, 42)
    qr = rrq.rotate(q[None], 42)[0]
    truth = float(np.dot(qr, r[0]))
    est = []
    for _ in range(4000):
        s = rg.standard_normal((d, d))
        v = s @ r[0]
        packed = np.packbits((v > 0).astype(np.uint8)[None], axis=1, bitorder="little")
        est.append(qjl.estimate_residual_dot(qr, s, packed, np.array([np.linalg.norm(r[0])]))[0])
    est = np.array(est)
    assert abs(est.mean() - truth) < 4 * est.std() / math.sqrt(est.size)
    # the residual chain corrects the MSE shrinkage on average
    assert np.linalg.norm(r[0]) > 0


# ---------------------------------------------------------- other GGML block types
def _ggml_inputs(name):
    j = np.arange(32)
    if name == "ramp16":
        return (j % 16) * 0.25 - 2.0
    if name == "ramp32":
        return j * 0.125 - 2.0
    if name == "halves":
        x = np.zeros(32)
        x[:6] = [127.0, 0.5, -0.5, 1.5, -2.5, 2.5]
        return x
    return _q4_inputs(name)


def test_ggml_hand_worked_blocks():
    lines = _golden_lines("ggml_blocks.txt")
    assert {ln.split("|")[0].strip() for ln in lines} == set(ggml_blocks.FORMATS)
    for ln in lines:
        fmt, name, hexbytes = (p.strip() for p in ln.split("|"))
        want = bytes.fromhex(hexbytes.replace(" ", ""))
        assert len(want) == ggml_blocks.BLOCK_BYTES[fmt], (fmt, name)
        enc = ggml_blocks.encode(_ggml_inputs(name)[None], 0, fmt, rotate_first=False)
        assert bytes(enc.blocks[0]) == want, (fmt, name, enc.blocks[0].tobytes().hex())


@pytest.mark.parametrize("fmt", ggml_blocks.FORMATS)
def test_ggml_grid_round_trip_exact(fmt):
    """Inputs on each type's own grid (step 2^-k, range fixed by the block) come back exactly."""
    rg = np.random.default_rng(5)
    n, d = 40, 128
    nb = d // 32
    if fmt in ("q4_1", "q5_1"):
        levels = 15 if fmt == "q4_1" else 31
        step = 2.0 ** rg.integers(-6, 2, size=(n, nb, 1))
        lo = rg.integers(-64, 64, size=(n, nb, 1)) * step
        q = rg.integers(0, levels + 1, size=(n, nb, 32))
        q[:, :, 0], q[:, :, 1] = 0, levels  # the block spans the whole range
        x = lo + q * step
    elif fmt == "q5_0":
        step = 2.0 ** rg.integers(-6, 2, size=(n, nb, 1))
        q = rg.integers(1, 32, size=(n, nb, 32))
        q[:, :, 0] = 0  # the first element of largest magnitude is -16 steps
        x = (q - 16) * step
    else:
        step = 2.0 ** rg.integers(-6, 2, size=(n, nb, 1))
        q = rg.integers(-126, 127, size=(n, nb, 32))
        q[:, :, 3] = 127
        x = q * step
    x = x.reshape(n, d)
    enc = ggml_blocks.encode(x, 0, fmt, rotate_first=False)
    assert np.array_equal(ggml_blocks.decode_exact(enc.blocks, d, 0, fmt, rotate_first=False), x)


@pytest.mark.parametrize("fmt", ggml_blocks.FORMATS)
def test_ggml_rotation_equivalence_and_error_bound(fmt):
    """rotate = 1 encodes Πx exactly as rotate = 0 encodes it; every decoded block value
    lies within half a step (plus the fp16 rounding of the stored scalars) of its input."""
    rg = np.random.default_rng(6)
    x = rg.standard_normal((30, 128)) * rg.uniform(0.1, 10, size=(30, 1))
    e1 = ggml_blocks.encode(x, 42, fmt, rotate_first=True)
    e0 = ggml_blocks.encode(rrq.rotate(x, 42), 0, fmt, rotate_first=False)
    assert np.array_equal(e1.blocks, e0.blocks)
    y = rrq.rotate(x, 42)
    v = ggml_blocks.dequantize(e1.blocks, 128, fmt)
    scale, mn, q = ggml_blocks.parse_blocks(e1.blocks, 128, fmt)
    step = np.repeat(np.abs(scale), 32, axis=1)
    # the clamp of the top code (q5_0, q4_0-like) costs up to one step on the
    # largest element of the opposite sign; everything else is within half a step
    slack = 1.0 if fmt == "q5_0" else 0.5
    err = np.abs(v - y)
    bound = slack * step + 2e-3 * np.repeat(np.max(np.abs(y.reshape(30, 4, 32)), axis=2), 32, axis=1)
    assert np.all(err <= bound)
    back = ggml_blocks.decode_exact(e1.blocks, 128, 42, fmt, rotate_first=True)
    assert np.allclose(rrq.rotate(back, 42), v)


def test_ggml_q8_rounds_half_away_from_zero_and_q4_1_matches_q4_0_on_symmetric_grids():
    x = np.zeros((1, 32))
    x[0, :4] = [127.0, 126.5, -126.5, -0.5]
    enc = ggml_blocks.encode(x, 0, "q8_0", rotate_first=False)
    assert enc.q[0, :4].tolist() == [127, 127, -127, -1]
    # both types reproduce a block whose values sit on their shared grid exactly
    g = ((np.arange(32) * 5) % 16 - 8) * 0.5
    g[0], g[1] = -4.0, 3.5
    e40 = q4_0.encode(g[None], 0, rotate_first=False)
    e41 = ggml_blocks.encode(g[None], 0, "q4_1", rotate_first=False)
    assert np.array_equal(q4_0.decode_exact(e40.blocks, 32, 0, rotate_first=False), g[None])
    assert np.array_equal(ggml_blocks.decode_exact(e41.blocks, 32, 0, "q4_1", rotate_first=False), g[None])


def test_ggml_signed_zero_rules():
    """A block of −0: the absmax types take the scale from +0 (Δ = +0/−16 = −0, fp16
    8000), the min/max types keep the first extreme in index order (here −0)."""
    x = np.full((1, 32), -0.0)
    b50 = ggml_blocks.encode(x, 0, "q5_0", rotate_first=False).blocks[0]
    assert b50[:2].tobytes() == b"\x00\x80"
    b41 = ggml_blocks.encode(x, 0, "q4_1", rotate_first=False).blocks[0]
    assert b41[:4].tobytes() == b"\x00\x00\x00\x80"
    x[0, 0] = 0.0  # +0 first, then −0: the min is the first, +0
    b41 = ggml_blocks.encode(x, 0, "q4_1", rotate_first=False).blocks[0]
    assert b41[:4].tobytes() == b"\x00\x00\x00\x00"


def test_q4_0_block_of_negative_zeros_stores_minus_zero_scale():
    """A block of −0: the scale comes from +0 (Δ = +0/−8 = −0, fp16 8000), every q = 8."""
    enc = q4_0.encode(np.full((1, 32), -0.0), 0, rotate_first=False)
    assert enc.blocks[0].tobytes() == bytes.fromhex("0080" + "88" * 16)



def test_qjl_unbiased_scores_average_to_the_true_inner_product():
    """scores_unbiased averaged over independent Gaussian projections S equals
    scale·<q, x> (the MSE score alone is biased low), for every head and token."""
    d, hq, hkv, t_len = 16, 4, 2, 3
    rg = np.random.default_rng(21)
    x = rg.standard_normal((t_len * hkv, d)) * 2.0
    q = rg.standard_normal((hq, d))
    g = np.arange(hq) // (hq // hkv)
    truth = 0.5 * np.einsum("hi,thi->ht", q, x.reshape(t_len, hkv, d)[:, g, :])
    acc, acc2, n = 0.0, 0.0, 3000
    for _ in range(n):
        s = rg.standard_normal((d, d))
        enc = qjl.encode(x, 2, 7, s)
        sc = qjl.scores_unbiased(q, enc.enc.packed, enc.enc.norms, enc.bits, enc.rnorm.astype(np.float64),
                                 t_len, hkv, d, 2, 7, s, scale=0.5)
        acc, acc2 = acc + sc, acc2 + sc * sc
    mean = acc / n
    sem = np.sqrt(np.maximum(acc2 / n - mean * mean, 0) / n)
    assert np.all(np.abs(mean - truth) < 4.5 * sem + 1e-9)
    mse_only = rrq.scores(q, enc.enc.packed, enc.enc.norms, t_len, hkv, d, 2, 7, scale=0.5)
    # the MSE part is the same for every S; the unbiased score differs from it by the estimate
    assert np.allclose(sc - mse_only,
                       np.stack([0.5 * qjl.estimate_residual_dot(rrq.rotate(q, 7)[h], s, enc.bits.reshape(t_len, hkv, 2)[:, g[h]],
                                                                  enc.rnorm.reshape(t_len, hkv)[:, g[h]]) for h in range(hq)]))



# ----------------------------------------------------- attention over a quantised cache
def _att_cache(t_len, hkv, d, seed_k, seed_v, rg):
    k = rg.standard_normal((t_len * hkv, d)) * 1.5
    v = rg.standard_normal((t_len * hkv, d)) * 0.8
    ek = rrq.encode(k, 4, seed_k)
    ev = rrq.encode(v, 4, seed_v)
    return ek, ev


def test_attention_single_token_returns_its_value():
    rg = np.random.default_rng(40)
    d, hkv, hq = 32, 2, 4
    ek, ev = _att_cache(1, hkv, d, 3, 5, rg)
    q = rg.standard_normal((hq, d))
    out = attention.decode_attention(q, ek.packed, ek.norms, ev.packed, ev.norms, 1, hkv, d, 4, 4, 3, 5)
    v_hat = rrq.decode_exact(ev.packed, ev.norms, 4, d, 5)
    for h in range(hq):
        assert np.allclose(out[h], v_hat[h // 2], rtol=0, atol=1e-12)


def test_attention_zero_query_is_the_mean_value_and_order_free():
    rg = np.random.default_rng(41)
    d, hkv, hq, t_len = 32, 2, 2, 7
    ek, ev = _att_cache(t_len, hkv, d, 3, 5, rg)
    out = attention.decode_attention(np.zeros((hq, d)), ek.packed, ek.norms, ev.packed, ev.norms,
                                     t_len, hkv, d, 4, 4, 3, 5)
    v_hat = rrq.decode_exact(ev.packed, ev.norms, 4, d, 5).reshape(t_len, hkv, d)
    assert np.allclose(out[0], v_hat[:, 0].mean(axis=0), atol=1e-12)
    assert np.allclose(out[1], v_hat[:, 1].mean(axis=0), atol=1e-12)
    q = rg.standard_normal((hq, d))
    perm = rg.permutation(t_len)
    rows = (perm[:, None] * hkv + np.arange(hkv)[None, :]).ravel()
    a = attention.decode_attention(q, ek.packed, ek.norms, ev.packed, ev.norms, t_len, hkv, d, 4, 4, 3, 5)
    b = attention.decode_attention(q, ek.packed[rows], ek.norms[rows], ev.packed[rows], ev.norms[rows],
                                   t_len, hkv, d, 4, 4, 3, 5)
    assert np.allclose(a, b, atol=1e-12)


def test_attention_large_scale_picks_the_top_scoring_token():
    rg = np.random.default_rng(42)
    d, hkv, hq, t_len = 32, 1, 1, 9
    ek, ev = _att_cache(t_len, hkv, d, 3, 5, rg)
    q = rg.standard_normal((hq, d))
    s = rrq.scores(q, ek.packed, ek.norms, t_len, hkv, d, 4, 3)
    top = int(np.argmax(s[0]))
    out = attention.decode_attention(q, ek.packed, ek.norms, ev.packed, ev.norms, t_len, hkv, d, 4, 4,
                                     3, 5, scale=1e4)
    v_hat = rrq.decode_exact(ev.packed, ev.norms, 4, d, 5)
    assert np.allclose(out[0], v_hat[top], atol=1e-9)
