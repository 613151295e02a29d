"""Plant plausible mistakes in the CPU oracle and check that the pins catch each one.

Every case patches one oracle function with a typical slip (transposed operand,
dropped normalisation, wrong sign, wrong index or bit order, wrong tie rule,
wrong constant) and asserts that at least one pin test from
``test_oracle_pins`` fails.  Nothing here touches a GPU.
"""

from __future__ import annotations

import math

import numpy as np
import pytest

import oracle.codebook as ocb
import oracle.ggml_blocks as ogg
import oracle.hadamard as oh
import oracle.q4_0 as oq4
import oracle.qjl as oqjl
import oracle.rrq as orrq
from tests import test_oracle_pins as pins


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_mutation_signs_after_transform(monkeypatch):
    """Π = D·H/√d instead of H·D/√d."""
    good = oh.rotation_matrix

    def bad(seed, d):
        h = oh.sylvester(d)
        s = oh.rotation_signs(seed, d)
        return s[:, None] * h / math.sqrt(d)

    monkeypatch.setattr(oh, "rotation_matrix", bad)
    monkeypatch.setattr(orrq, "rotation_matrix", bad)
    assert _fails(pins.test_rotation_is_orthogonal_and_signs_first, 128)
    monkeypatch.setattr(oh, "rotation_matrix", good)


def test_mutation_missing_normalisation(monkeypatch):
    def bad(seed, d):
        return oh.sylvester(d) * oh.rotation_signs(seed, d)[None, :]

    monkeypatch.setattr(oh, "rotation_matrix", bad)
    monkeypatch.setattr(orrq, "rotation_matrix", bad)
    assert _fails(pins.test_rotation_is_orthogonal_and_signs_first, 64)


def test_mutation_decode_with_pi_instead_of_pi_transpose(monkeypatch):
    good = orrq.rotate

    def bad(x, seed, inverse=False):
        return good(x, seed, inverse=False)

    monkeypatch.setattr(orrq, "rotate", bad)
    assert _fails(pins.test_round_trip_nmse_matches_lloyd_max_distortion, 4)


def test_mutation_tie_rule(monkeypatch):
    good = np.searchsorted

    def bad_encode(x, bits, seed, levels=None):
        enc = good_encode(x, bits, seed, levels)
        tau = ocb.thresholds(ocb.lloyd_max(bits) if levels is None else levels)
        enc.codes = good(tau, enc.u.ravel(), side="right").reshape(enc.codes.shape)
        enc.packed = orrq.pack_codes(enc.codes, bits)
        return enc

    good_encode = orrq.encode
    monkeypatch.setattr(orrq, "encode", bad_encode)
    assert _fails(pins.test_zero_vector_and_exact_ties)


def test_mutation_msb_first_packing(monkeypatch):
    good = orrq.pack_codes

    def bad(codes, bits):
        codes = np.asarray(codes, dtype=np.int64)
        n, d = codes.shape
        planes = ((codes[:, :, None] >> np.arange(bits)[None, None, :]) & 1).astype(np.uint8)
        return np.packbits(planes.reshape(n, d * bits), axis=1, bitorder="big")

    monkeypatch.setattr(orrq, "pack_codes", bad)
    assert _fails(pins.test_pack_matches_bitwise_reference, 4)
    monkeypatch.setattr(orrq, "pack_codes", good)


def test_mutation_centroid_sign(monkeypatch):
    """Lloyd update with φ(τ_k) − φ(τ_{k−1}) (sign flipped) must miss the page values."""
    ocb._lloyd_max.cache_clear()
    good_phi = ocb._phi
    monkeypatch.setattr(ocb, "_phi", lambda x: -good_phi(x))
    try:
        assert _fails(pins.test_codebook_page_values)
    except (ValueError, ZeroDivisionError, OverflowError):
        pass  # a diverging iteration is also caught
    finally:
        monkeypatch.setattr(ocb, "_phi", good_phi)
        ocb._lloyd_max.cache_clear()


def test_mutation_q4_0_nibble_order(monkeypatch):
    good = oq4.encode

    def bad(x, seed, rotate_first=True):
        enc = good(x, seed, rotate_first)
        b = enc.blocks.reshape(enc.blocks.shape[0], -1, 18).copy()
        b[:, :, 2:] = ((b[:, :, 2:] & 0x0F) << 4) | (b[:, :, 2:] >> 4)
        enc.blocks = b.reshape(enc.blocks.shape)
        return enc

    monkeypatch.setattr(oq4, "encode", bad)
    assert _fails(pins.test_q4_0_hand_worked_blocks)


def test_mutation_q4_0_unsigned_max(monkeypatch):
    """Using +max|x| instead of the signed extreme for Δ."""
    def bad(x, seed, rotate_first=True):
        x = np.asarray(x, dtype=np.float64)
        y = orrq.rotate(x, seed) if rotate_first else x
        flipped = good(np.abs(y) * np.sign(y + 0.0) * 1.0, 0, rotate_first=False)
        m = np.abs(y.reshape(y.shape[0], -1, 32)).max(axis=2)
        delta = (m.astype(np.float32) / np.float32(-8.0))
        b = flipped.blocks.reshape(y.shape[0], -1, 18).copy()
        dh = delta.astype(np.float16).view(np.uint16)
        b[:, :, 0] = dh & 0xFF
        b[:, :, 1] = dh >> 8
        flipped.blocks = b.reshape(flipped.blocks.shape)
        return flipped

    good = oq4.encode
    monkeypatch.setattr(oq4, "encode", bad)
    assert _fails(pins.test_q4_0_hand_worked_blocks)


@pytest.mark.parametrize("factor", [1.0, math.pi / 2])
def test_mutation_qjl_constant(monkeypatch, factor):
    """Dropping √(π/2) (or squaring it) biases the estimator."""
    good = oqjl.estimate_residual_dot

    def bad(q_rot, s_matrix, packed_signs, rnorm):
        return good(q_rot, s_matrix, packed_signs, rnorm) / math.sqrt(math.pi / 2) * factor

    monkeypatch.setattr(oqjl, "estimate_residual_dot", bad)
    assert _fails(pins.test_qjl_estimator_unbiased_monte_carlo)


def test_mutation_q8_0_rounds_half_to_even(monkeypatch):
    """q8_0 codes with numpy's round-half-to-even instead of halves away from zero."""
    good = ogg.block_decisions

    def bad(y32, fmt, pick=None):
        q, s32, m32, margin = good(y32, fmt, pick)
        if fmt == "q8_0":
            inv = np.where(s32 != 0, np.float32(1.0) / np.where(s32 != 0, s32, 1), 0).astype(np.float32)
            q = np.round((np.asarray(y32, np.float32) * inv[..., None]).astype(np.float32)).astype(np.int64)
        return q, s32, m32, margin

    monkeypatch.setattr(ogg, "block_decisions", bad)
    assert _fails(pins.test_ggml_hand_worked_blocks)


def test_mutation_q5_high_bits_reversed(monkeypatch):
    """The q5 high-bit word with bit 31 − j instead of bit j."""
    good = ogg.serialize

    def bad(fmt, q, scale32, min32):
        if fmt in ("q5_0", "q5_1"):
            q = q[..., ::-1].copy() & 16 | (q & 15)
        return good(fmt, q, scale32, min32)

    monkeypatch.setattr(ogg, "serialize", bad)
    assert _fails(pins.test_ggml_hand_worked_blocks)


def test_mutation_q4_1_min_and_scale_swapped(monkeypatch):
    """q4_1 / q5_1 with the min stored before the scale."""
    good = ogg.serialize

    def bad(fmt, q, scale32, min32):
        if fmt in ("q4_1", "q5_1"):
            return good(fmt, q, min32, scale32)
        return good(fmt, q, scale32, min32)

    monkeypatch.setattr(ogg, "serialize", bad)
    assert _fails(pins.test_ggml_hand_worked_blocks)


def test_mutation_q5_0_scale_from_unsigned_max(monkeypatch):
    """q5_0 with Δ = max|y|/−16 (the sign of the largest element dropped)."""
    good = ogg.block_decisions

    def bad(y32, fmt, pick=None):
        if fmt != "q5_0":
            return good(y32, fmt, pick)
        y32 = np.asarray(y32, np.float32)
        a = np.max(np.abs(y32), axis=-1)
        delta = (a / np.float32(-16.0)).astype(np.float32)
        inv = np.where(delta != 0, np.float32(1.0) / np.where(delta != 0, delta, 1), 0).astype(np.float32)
        r = ((y32 * inv[..., None]).astype(np.float32) + np.float32(16.5)).astype(np.float32)
        q = np.clip(np.floor(r), 0, 31).astype(np.int64)
        return q, delta, np.zeros_like(delta), np.zeros(y32.shape)

    monkeypatch.setattr(ogg, "block_decisions", bad)
    assert _fails(pins.test_ggml_hand_worked_blocks)


def test_mutation_attention_values_decoded_with_the_key_rotation(monkeypatch):
    """v̂ decoded with the key seed instead of the value seed."""
    import oracle.attention as oatt
    good = oatt.decode_attention

    def bad(q, kp, kn, vp, vn, t_len, hkv, d, kb, vb, ks, vs, *a, **kw):
        return good(q, kp, kn, vp, vn, t_len, hkv, d, kb, vb, ks, ks, *a, **kw)

    monkeypatch.setattr(oatt, "decode_attention", bad)
    assert _fails(pins.test_attention_single_token_returns_its_value)


def test_mutation_attention_softmax_over_heads(monkeypatch):
    """The softmax normalised over the query heads instead of the tokens."""
    import oracle.attention as oatt

    def bad(q, kp, kn, vp, vn, t_len, hkv, d, kb, vb, ks, vs, kl=None, vl=None, scale=1.0):
        q = np.asarray(q, np.float64)
        s = orrq.scores(q, kp, kn, t_len, hkv, d, kb, ks, kl, scale)
        w = np.exp(s - s.max(axis=0, keepdims=True))
        p = w / w.sum(axis=0, keepdims=True)
        v_hat = orrq.decode_exact(vp, vn, vb, d, vs, vl).reshape(t_len, hkv, d)
        return np.stack([p[h] @ v_hat[:, orrq.kv_group(h, q.shape[0], hkv), :] for h in range(q.shape[0])])

    monkeypatch.setattr(oatt, "decode_attention", bad)
    assert _fails(pins.test_attention_zero_query_is_the_mean_value_and_order_free)


def _unbiased_with(residual_query, group_of):
    """scores_unbiased with the residual term's query and kv group replaced."""

    def bad(q, packed, norms, qjl_bits, rnorm, t_len, hkv, d, bits, seed, s_matrix, levels=None,
            scale=1.0):
        q = np.asarray(q, np.float64)
        hq = q.shape[0]
        out = orrq.scores(q, packed, norms, t_len, hkv, d, bits, seed, levels, scale)
        qr = residual_query(q, seed)
        qb = np.asarray(qjl_bits, dtype=np.uint8).reshape(t_len, hkv, d // 8)
        rn = np.asarray(rnorm, np.float64).reshape(t_len, hkv)
        for h in range(hq):
            g = group_of(h, hq, hkv)
            out[h] += scale * oqjl.estimate_residual_dot(qr[h], s_matrix, qb[:, g, :], rn[:, g])
        return out

    return bad


def test_mutation_unbiased_residual_with_the_unrotated_query(monkeypatch):
    """The QJL term dotted with S·q instead of S·Πq (the sketch lives in the rotated domain)."""
    monkeypatch.setattr(oqjl, "scores_unbiased", _unbiased_with(lambda q, seed: q, orrq.kv_group))
    assert _fails(pins.test_qjl_unbiased_scores_average_to_the_true_inner_product)


def test_mutation_unbiased_residual_with_the_wrong_kv_group(monkeypatch):
    """The QJL term of head h taken from kv head h mod Hkv instead of ⌊h·Hkv/Hq⌋."""
    monkeypatch.setattr(oqjl, "scores_unbiased",
                        _unbiased_with(orrq.rotate, lambda h, hq, hkv: h % hkv))
    assert _fails(pins.test_qjl_unbiased_scores_average_to_the_true_inner_product)


def test_mutation_unbiased_residual_subtracted(monkeypatch):
    """The residual estimate subtracted instead of added."""
    monkeypatch.setattr(oqjl, "scores_unbiased",
                        _unbiased_with(lambda q, seed: -orrq.rotate(q, seed), orrq.kv_group))
    assert _fails(pins.test_qjl_unbiased_scores_average_to_the_true_inner_product)


def test_unbiased_harness_unmutated_passes(monkeypatch):
    """Control: the harness above with the right query and group passes the pin, so the
    three failures come from the planted slips alone."""
    monkeypatch.setattr(oqjl, "scores_unbiased", _unbiased_with(orrq.rotate, orrq.kv_group))
    assert not _fails(pins.test_qjl_unbiased_scores_average_to_the_true_inner_product)


def _attention_with(group_of, use_scale, key_seed_of):
    """decode_attention with the kv group map, the score scale or the key rotation seed replaced."""

    def bad(q, kp, kn, vp, vn, t_len, hkv, d, kb, vb, ks, vs, kl=None, vl=None, scale=1.0):
        q = np.asarray(q, np.float64)
        hq = q.shape[0]
        s = orrq.scores(q, kp, kn, t_len, hkv, d, kb, key_seed_of(ks, vs), kl, scale if use_scale else 1.0)
        w = np.exp(s - s.max(axis=1, keepdims=True))
        p = w / w.sum(axis=1, keepdims=True)
        v_hat = orrq.decode_exact(vp, vn, vb, d, vs, vl).reshape(t_len, hkv, d)
        return np.stack([p[h] @ v_hat[:, group_of(h, hq, hkv), :] for h in range(hq)])

    return bad


_ATT_PINS = (lambda: pins.test_attention_single_token_returns_its_value(),
             lambda: pins.test_attention_zero_query_is_the_mean_value_and_order_free(),
             lambda: pins.test_attention_large_scale_picks_the_top_scoring_token())


def _any_pin_fails():
    return any(_fails(p) for p in _ATT_PINS)


@pytest.mark.parametrize("slip", ["group", "scale", "key_seed"])
def test_mutation_attention_slips(monkeypatch, slip):
    """Head h reading kv head h mod Hkv; the score scale dropped; the scores taken
    under the value rotation instead of the key rotation."""
    import oracle.attention as oatt
    group_of = (lambda h, hq, hkv: h % hkv) if slip == "group" else orrq.kv_group
    key_seed_of = (lambda ks, vs: vs) if slip == "key_seed" else (lambda ks, vs: ks)
    monkeypatch.setattr(oatt, "decode_attention", _attention_with(group_of, slip != "scale", key_seed_of))
    assert _any_pin_fails()


def test_attention_harness_unmutated_passes(monkeypatch):
    """Control: the harness with the right map, scale and seed passes every attention pin."""
    import oracle.attention as oatt
    monkeypatch.setattr(oatt, "decode_attention",
                        _attention_with(orrq.kv_group, True, lambda ks, vs: ks))
    assert not _any_pin_fails()


# ---------------------------------------------------------------- DRIVE
def _drive_encode_with(sign_rule, stored_factor):
    """drive_encode with the sign rule or the stored scale factor replaced."""
    import oracle.sphere as osp

    def bad(x, seed, unbiased):
        x = np.asarray(x, np.float64)
        d = x.shape[-1]
        rx = orrq.rotate(x, seed)
        with np.errstate(invalid="ignore", divide="ignore"):
            s = osp.drive_scale_unbiased(x, rx) if unbiased else osp.drive_scale_biased(rx)
        s = np.where(np.sum(np.abs(rx), axis=-1) > 0, s, 0.0)
        signs = sign_rule(rx).astype(np.int64)
        stored = (s * stored_factor(d)).astype(np.float32)
        return osp.DriveEncoded(signs, orrq.pack_codes(signs, 1), s, stored, rx)

    return bad


def test_mutation_drive_biased_scale_with_the_two_norm(monkeypatch):
    """S = ‖R(x)‖₂/d instead of ‖R(x)‖₁/d."""
    import oracle.sphere as osp
    monkeypatch.setattr(osp, "drive_scale_biased",
                        lambda rx: np.linalg.norm(np.asarray(rx, np.float64), axis=-1) / np.shape(rx)[-1])
    assert _fails(pins.test_drive_biased_scale_is_mse_optimal, 16)


def test_mutation_drive_unbiased_scale_with_the_two_norm(monkeypatch):
    """S = ‖x‖₂²/‖R(x)‖₂ instead of ‖x‖₂²/‖R(x)‖₁."""
    import oracle.sphere as osp

    def bad(x, rx):
        x, rx = np.asarray(x, np.float64), np.asarray(rx, np.float64)
        return np.sum(x * x, axis=-1) / np.linalg.norm(rx, axis=-1)

    monkeypatch.setattr(osp, "drive_scale_unbiased", bad)
    assert _fails(pins.test_drive_unbiased_scale, 8)


def test_mutation_drive_zero_takes_plus_one(monkeypatch):
    """sign(0) = +1 in the encoder (the decoder and the b-bit rule keep −1)."""
    import oracle.sphere as osp
    monkeypatch.setattr(osp, "drive_encode", _drive_encode_with(lambda rx: rx >= 0, math.sqrt))
    assert _fails(pins.test_drive_zero_coordinates_take_the_minus_one_sign)


def test_mutation_drive_stored_without_sqrt_d(monkeypatch):
    """The stored per-vector value S instead of S·√d."""
    import oracle.sphere as osp
    monkeypatch.setattr(osp, "drive_encode", _drive_encode_with(lambda rx: rx > 0, lambda d: 1.0))
    assert _fails(pins.test_drive_encode_through_the_one_bit_decoder, False)


def test_drive_harness_unmutated_passes(monkeypatch):
    """Control: the encoder harness with the right sign rule and factor passes both pins."""
    import oracle.sphere as osp
    monkeypatch.setattr(osp, "drive_encode", _drive_encode_with(lambda rx: rx > 0, math.sqrt))
    assert not _fails(pins.test_drive_zero_coordinates_take_the_minus_one_sign)
    assert not _fails(pins.test_drive_encode_through_the_one_bit_decoder, False)
    assert not _fails(pins.test_drive_encode_through_the_one_bit_decoder, True)
