"""Comparison helpers for GPU-vs-oracle parity (the tolerances, in one place).

Tolerances (stated for this hot path, and derived where they were not):

* rotated fp32 values: max |y_gpu − y_oracle| ≤ 1e-5·‖x‖ per vector;
* reconstructions: ‖x̂_gpu − x̂_oracle‖₂ ≤ 2e-3·‖x‖₂ per vector, with the GPU
  decoding the oracle's codes so encode exemptions cannot leak in;
* codes and packed bytes: bit-exact, except a code may differ by one step
  when the oracle's normalised coordinate u lies within 1e-5 (σ = 1 in u
  units) of the threshold between the two codes; such exempt mismatches
  must be fewer than 1e-4 of all codes;
* scores: |s_gpu − s_oracle| ≤ 1e-3·‖q‖·‖k̂‖·|scale| (per-element relative error
  is undefined near 0, so the Cauchy–Schwarz scale of the score is used);
* norms: relative error ≤ d·2⁻²⁴ (worst case of an fp32 sum of d squares);
* decode attention: per query head, ‖out_gpu − out_oracle‖ ≤ 2e-3·Σ_t p_t·‖v̂_t‖
  with p the oracle's softmax weights (the reconstruction tolerance carried
  through the convex combination by the triangle inequality).
"""

from __future__ import annotations

import numpy as np

EXEMPT_BAND = 1e-5
EXEMPT_RATE = 1e-4


def unpack_codes(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).reshape(-1, d * bits // 8)
    n = packed.shape[0]
    flat = np.unpackbits(packed, axis=1, bitorder="little")[:, : d * bits].reshape(n, d, bits)
    return (flat.astype(np.int64) << np.arange(bits)[None, None, :]).sum(axis=2)


def code_mismatches(gpu_codes: np.ndarray, orc_codes: np.ndarray, u: np.ndarray,
                    tau: np.ndarray, band: float = EXEMPT_BAND):
    """-> (exempt count, non-exempt count, total).  Codes as [N, d] integer arrays."""
    gpu_codes = np.asarray(gpu_codes, dtype=np.int64)
    orc_codes = np.asarray(orc_codes, dtype=np.int64)
    diff = gpu_codes != orc_codes
    total = gpu_codes.size
    if not diff.any():
        return 0, 0, total
    g, o, uu = gpu_codes[diff], orc_codes[diff], u[diff]
    step = np.abs(g - o) == 1
    lo = np.minimum(g, o)
    near = np.zeros_like(step)
    near[step] = np.abs(uu[step] - tau[lo[step]]) < band
    exempt = int(np.sum(step & near))
    return exempt, int(diff.sum()) - exempt, total


def assert_codes_match(gpu_codes, orc_codes, u, tau, what=""):
    exempt, bad, total = code_mismatches(gpu_codes, orc_codes, u, tau)
    assert bad == 0, f"{what}: {bad} code mismatches outside the 1e-5 boundary band"
    assert exempt < EXEMPT_RATE * total, f"{what}: {exempt} exempt mismatches of {total}"
    return exempt


def assert_rotated_close(y_gpu, y_orc, x_norm, what=""):
    err = np.max(np.abs(np.asarray(y_gpu, np.float64) - y_orc), axis=1)
    bound = 1e-5 * np.asarray(x_norm, np.float64)
    ok = err <= bound + 1e-30
    assert ok.all(), f"{what}: rotated error {err[~ok][:3]} > {bound[~ok][:3]}"


def assert_reconstruction_close(x_gpu, x_orc, x_norm, what="", rel=2e-3):
    err = np.sqrt(np.sum((np.asarray(x_gpu, np.float64) - x_orc) ** 2, axis=1))
    bound = rel * np.asarray(x_norm, np.float64)
    ok = err <= bound + 1e-30
    assert ok.all(), f"{what}: reconstruction error {err[~ok][:3]} > {bound[~ok][:3]}"


def assert_norms_close(n_gpu, n_orc, d, what=""):
    n_gpu = np.asarray(n_gpu, np.float64)
    n_orc = np.asarray(n_orc, np.float64)
    tol = d * 2.0 ** -24
    rel = np.abs(n_gpu - n_orc) / np.maximum(n_orc, 1e-300)
    rel[n_orc == 0] = np.abs(n_gpu[n_orc == 0])
    assert np.all(rel <= tol), f"{what}: norm relative error {rel.max()} > {tol}"


def assert_scores_close(s_gpu, s_orc, cs_scale, scale=1.0, what=""):
    err = np.abs(np.asarray(s_gpu, np.float64) - s_orc)
    bound = 1e-3 * cs_scale * abs(scale)
    ok = err <= bound + 1e-30
    assert ok.all(), f"{what}: {np.sum(~ok)} scores off; worst ratio {np.max(err / np.maximum(bound, 1e-300))}"


def attention_bound(p, v_packed, v_norms, t_len, hkv, d, v_bits, v_seed, v_levels=None,
                    rel=2e-3):
    """rel·Σ_t p[h,t]·‖v̂_{t,g(h)}‖ per query head, v̂ the oracle's value reconstructions."""
    from oracle import rrq as orc
    v_hat = orc.decode_exact(v_packed, v_norms, v_bits, d, v_seed, v_levels).reshape(t_len, hkv, d)
    vnorm = np.linalg.norm(v_hat, axis=2)  # [T, hkv]
    hq = p.shape[0]
    g = np.array([orc.kv_group(h, hq, hkv) for h in range(hq)])
    return rel * np.einsum("ht,ht->h", p, vnorm[:, g].T)
