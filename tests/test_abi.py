"""The C ABI without a GPU: the library loads, exports every declared symbol,
validates arguments before any launch, and its host-side helpers (codebook,
QJL matrix) agree with the oracle.  No kernel is launched here."""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

from oracle import codebook as ocb
from oracle import rng as orng
from random_rotation_kv_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rrq.h")


def _declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(rrq_\w+)\s*\(", text)))


def test_library_loads_and_exports_every_declared_symbol():
    lib = B.lib()
    declared = _declared_symbols()
    assert len(declared) >= 10
    for name in declared:
        assert hasattr(lib, name), name
    # the binding declares exactly the header's entry points
    assert sorted(B.SIGNATURES) == declared


def test_format_version_and_strerror():
    assert B.rrq_format_version() == 1
    for st in range(4):
        assert len(B.strerror(st)) > 0
    assert B.strerror(99) == "unknown status"


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_default_codebook_matches_oracle(bits):
    c = B.rrq_codebook(bits).astype(np.float64)
    o = ocb.lloyd_max(bits)
    assert np.all(np.abs(c - o) <= 2 ** -23 * np.abs(o))  # float rounding of the same levels
    assert np.array_equal(c, -c[::-1])


def test_codebook_rejects_bad_bits():
    lib = B.lib()
    buf = (ctypes.c_float * 32)()
    for bits in (0, 5, -1):
        assert lib.rrq_codebook(bits, ctypes.cast(buf, ctypes.c_void_p)) == B.RRQ_ERR_INVALID
    assert lib.rrq_codebook(2, None) == B.RRQ_ERR_INVALID


@pytest.mark.parametrize("d", [64, 128])
def test_qjl_matrix_bit_exact_vs_oracle(d):
    lib = B.lib()
    host = np.zeros(d * d, dtype=np.uint16)
    assert lib.rrq_qjl_matrix(4242, d, ctypes.c_void_p(host.ctypes.data)) == B.RRQ_OK
    want = orng.bf16_bits(orng.qjl_gaussian(4242, d)).ravel()
    assert np.array_equal(host, want)
    assert lib.rrq_qjl_matrix(1, 100, ctypes.c_void_p(host.ctypes.data)) == B.RRQ_ERR_INVALID


# Fake, never-dereferenced device addresses: every call below must be rejected
# by validation before any CUDA call.
P = ctypes.c_void_p(0x10000)
P_MIS = ctypes.c_void_p(0x10002)


def test_encode_validation_before_launch():
    lib = B.lib()
    enc = lib.rrq_encode
    ok = dict(x=P, dt=B.RRQ_F16, n=8, d=128, bits=4)

    def call(**kw):
        a = {**ok, **kw}
        return enc(a["x"], a["dt"], a["n"], a["d"], a["bits"], 42, kw.get("cb"), P, P,
                   kw.get("S"), kw.get("qb"), kw.get("qn"), None)

    assert call(d=100) == B.RRQ_ERR_INVALID
    assert call(d=32) == B.RRQ_ERR_INVALID
    assert call(d=1024) == B.RRQ_ERR_INVALID
    assert call(bits=0) == B.RRQ_ERR_INVALID
    assert call(bits=5) == B.RRQ_ERR_INVALID
    assert call(dt=7) == B.RRQ_ERR_INVALID
    assert call(n=-1) == B.RRQ_ERR_INVALID
    assert call(x=ctypes.c_void_p(None)) == B.RRQ_ERR_INVALID
    assert call(x=P_MIS) == B.RRQ_ERR_INVALID
    bad_cb = (ctypes.c_float * 16)(*([0.0] * 16))  # not strictly ascending
    assert call(cb=ctypes.cast(bad_cb, ctypes.c_void_p)) == B.RRQ_ERR_INVALID
    nan_cb = (ctypes.c_float * 16)(*([float("nan")] + list(range(15))))
    assert call(cb=ctypes.cast(nan_cb, ctypes.c_void_p)) == B.RRQ_ERR_INVALID
    # QJL outputs must be given with S
    assert call(S=P, qb=None, qn=P) == B.RRQ_ERR_INVALID
    # n = 0 with valid arguments is a no-op that touches nothing
    assert call(n=0, x=ctypes.c_void_p(None)) == B.RRQ_OK


def test_other_entry_points_validate():
    lib = B.lib()
    assert lib.rrq_decode(P, P, 4, 100, 4, 0, None, P, B.RRQ_F16, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_decode(P, P, 4, 128, 4, 0, None, P, 9, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_decode(P, P_MIS, 4, 128, 4, 0, None, P, B.RRQ_F16, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_rotate(P, B.RRQ_F16, 4, 128, 0, 2, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_rotate(P_MIS, B.RRQ_F16, 4, 128, 0, 0, P, None) == B.RRQ_ERR_INVALID
    # scores: hq not a multiple of hkv, unsupported group, non-finite scale
    assert lib.rrq_qk_scores(P, 30, P, P, 16, 8, 128, 4, 0, None, 1.0, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_qk_scores(P, 48, P, P, 16, 3, 128, 4, 0, None, 1.0, P, None) == B.RRQ_ERR_UNSUPPORTED
    assert lib.rrq_qk_scores(P, 32, P, P, 16, 8, 128, 4, 0, None, float("inf"), P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_qk_scores(P, 32, P, P, 0, 8, 128, 4, 0, None, 1.0, P, None) == B.RRQ_OK
    assert lib.rrq_q4_0_rot(P, B.RRQ_F16, 4, 96, 0, 1, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_q4_0_rot(P, B.RRQ_F16, 4, 128, 0, 3, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_q4_0_rot_decode(P, 4, 128, 0, 1, P, 5, None) == B.RRQ_ERR_INVALID
    # attention: group sizes 1, 2, 4, 8 (at most 4 at d = 512); T must be at least 1;
    # a big enough workspace (every call here is refused before any launch)
    assert lib.rrq_attention_decode(P, 24, P, P, P, P, 16, 8, 128, 4, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_UNSUPPORTED
    assert lib.rrq_attention_decode(P, 64, P, P, P, P, 16, 8, 512, 2, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_UNSUPPORTED
    assert lib.rrq_attention_decode(P, 32, P, P, P, P, 16, 8, 96, 4, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_decode(P, 32, P, P, P, P, 16, 8, 128, 5, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_decode(P, 32, P, P, P, P, 16, 8, 64, 2, 0, None, 3, 1, None, 1.0, P, 64, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_decode(P, 32, P, P, P, P, 0, 8, 128, 4, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_decode(P, 32, P, P, P_MIS, P, 16, 8, 128, 4, 0, None, 4, 1, None, 1.0, P, 1 << 30, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_decode(P, 32, P, P, P, P, 16, 8, 128, 4, 0, None, 4, 1, None, 1.0, P, 16, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_attention_workspace_bytes(32, 8, 128, 4, 4, 1 << 17) > 0
    assert lib.rrq_attention_workspace_bytes(30, 8, 128, 4, 4, 16) == 0
    assert lib.rrq_attention_workspace_bytes(32, 8, 128, 4, 0, 16) == 0
    # the fused shape needs no score buffer; every other shape does (hq × T floats)
    assert lib.rrq_attention_workspace_bytes(32, 8, 128, 2, 2, 1 << 17) >= 32 * (1 << 17) * 4
    assert lib.rrq_attention_workspace_bytes(32, 8, 128, 4, 4, 1 << 17) < 32 * (1 << 17) * 4
    # unbiased scores: d other than 128 and odd group sizes are unsupported; S must be given
    assert lib.rrq_qk_scores_qjl(P, 32, P, P, P, P, P, 16, 8, 64, 2, 0, None, 1.0, P, None) == B.RRQ_ERR_UNSUPPORTED
    assert lib.rrq_qk_scores_qjl(P, 48, P, P, P, P, P, 16, 3, 128, 2, 0, None, 1.0, P, None) == B.RRQ_ERR_UNSUPPORTED
    assert lib.rrq_qk_scores_qjl(P, 32, P, P, P, P, None, 16, 8, 128, 2, 0, None, 1.0, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_qk_scores_qjl(P, 32, P, P, P_MIS, P, P, 16, 8, 128, 2, 0, None, 1.0, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_qk_scores_qjl(P, 32, P, P, P, P, P, 0, 8, 128, 2, 0, None, 1.0, P, None) == B.RRQ_OK
    # GGML block types: sizes, unknown types, bad rotate flag
    assert [lib.rrq_ggml_block_bytes(t) for t in (2, 3, 6, 7, 8, 1, 9)] == [18, 20, 22, 24, 34, 0, 0]
    assert lib.rrq_ggml_rot(P, B.RRQ_F16, 4, 128, 0, 1, 4, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_ggml_rot(P, B.RRQ_F16, 4, 128, 0, 2, 3, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_ggml_rot(P, B.RRQ_F16, 4, 96, 0, 1, 3, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_ggml_rot_decode(P, 5, 4, 128, 0, 1, P, B.RRQ_F16, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_ggml_rot_decode(P_MIS, 3, 4, 128, 0, 1, P, B.RRQ_F16, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_ggml_rot(ctypes.c_void_p(None), B.RRQ_F16, 0, 128, 0, 1, 8, P, None) == B.RRQ_OK
    # DRIVE: unbiased must be 0/1, d a supported size, scales 4-byte aligned
    assert lib.rrq_drive_encode(P, B.RRQ_F16, 4, 128, 0, 2, P, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_drive_encode(P, B.RRQ_F16, 4, 100, 0, 0, P, P, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_drive_encode(P, B.RRQ_F16, 4, 128, 0, 1, P, P_MIS, None) == B.RRQ_ERR_INVALID
    assert lib.rrq_drive_encode(ctypes.c_void_p(None), B.RRQ_F16, 0, 128, 0, 1, P, P, None) == B.RRQ_OK


@pytest.mark.parametrize("hq,hkv", [(32, 8), (8, 1), (16, 2), (32, 32), (64, 8)])
def test_attention_splits_fill_the_sms_in_one_wave(hq, hkv):
    """The token ranges per kv head that rrq_attention_workspace_bytes implies: one CTA
    per SM, rounded down so that hkv × ranges never exceeds the SM count (that of
    the visible device; 148, the library's default, when none is visible); a range
    per 12 tiles of 32 tokens (one per warp) at most; at least one."""
    import torch
    lib = B.lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    counters = (hkv * 4 + 255) // 256 * 256
    for t_len in (1, 100, 4096, 1 << 17, 1 << 20):
        ws = lib.rrq_attention_workspace_bytes(hq, hkv, 128, 4, 4, t_len)
        per_range = hq * 131 * 4
        assert (ws - counters) % per_range == 0
        s = (ws - counters) // per_range
        ntile = (t_len + 31) // 32
        assert s == max(1, min(sms // hkv, (ntile + 11) // 12))
        assert s * hkv <= max(sms, hkv)


@pytest.mark.parametrize("hq,hkv,d", [(32, 8, 64), (32, 8, 256), (8, 1, 512), (64, 8, 128)])
def test_general_attention_workspace(hq, hkv, d):
    """Shapes other than d = 128 with 4-bit K and V: counters (256-byte padded), the
    ranges' partial states (hq × ranges × (d + 2) floats, 256-byte padded), then the
    scores (hq × T floats); as many CTAs as the SMs hold at once (one to three each, by
    the occupancy of the value kernel for that d and V bit width: one when no device is
    visible), at most 444 ranges per kv head, at least 32 tokens per range, at least
    one range."""
    import torch
    lib = B.lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148
    counters = (hkv * 4 + 255) // 256 * 256
    for t_len, v_bits in ((1, 3), (100, 1), (4096, 2), (1 << 17, 3), (1 << 17, 4)):
        ws = lib.rrq_attention_workspace_bytes(hq, hkv, d, 2, v_bits, t_len)
        sizes = []
        for per_sm in (1, 2, 3):
            s = max(1, min(per_sm * sms // hkv, 444, (t_len + 31) // 32))
            sizes.append(counters + (hq * s * (d + 2) * 4 + 255) // 256 * 256 + hq * t_len * 4)
        assert ws in sizes, (ws, sizes)
        if not torch.cuda.is_available():
            assert ws == sizes[0]
