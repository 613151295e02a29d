"""Thin ctypes binding of librrq.so with the C ABI's names (argument marshalling only).

Every function checks that its tensors are contiguous CUDA tensors of the
right type, passes raw device pointers, sizes and torch's current CUDA stream
to the C entry point of the same name, and raises ``RRQError`` on a non-zero
status.  All arithmetic runs in the library's CUDA kernels; there is no CPU
path.  If ``librrq.so`` is missing the first call raises immediately.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librrq.so")

RRQ_OK, RRQ_ERR_INVALID, RRQ_ERR_CUDA, RRQ_ERR_UNSUPPORTED, RRQ_ERR_SCRATCH = 0, 1, 2, 3, 4
RRQ_F32, RRQ_F16, RRQ_BF16 = 0, 1, 2
DTYPE_CODE = {torch.float32: RRQ_F32, torch.float16: RRQ_F16, torch.bfloat16: RRQ_BF16}
# GGML block types (ggml's own type numbers), as in include/rrq.h
GGML_TYPES = {"q4_0": 2, "q4_1": 3, "q5_0": 6, "q5_1": 7, "q8_0": 8}

_c_i64 = ctypes.c_int64
_c_u64 = ctypes.c_uint64
_vp = ctypes.c_void_p
_int = ctypes.c_int
_fp = ctypes.POINTER(ctypes.c_float)

# name -> (restype, argtypes), mirroring include/rrq.h
SIGNATURES = {
    "rrq_format_version": (_int, []),
    "rrq_strerror": (ctypes.c_char_p, [_int]),
    "rrq_codebook": (_int, [_int, _vp]),
    "rrq_rotate": (_int, [_vp, _int, _c_i64, _int, _c_u64, _int, _vp, _vp]),
    "rrq_encode": (_int, [_vp, _int, _c_i64, _int, _int, _c_u64, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "rrq_decode": (_int, [_vp, _vp, _c_i64, _int, _int, _c_u64, _vp, _vp, _int, _vp]),
    "rrq_drive_encode": (_int, [_vp, _int, _c_i64, _int, _c_u64, _int, _vp, _vp, _vp]),
    "rrq_qk_scores": (_int, [_vp, _int, _vp, _vp, _c_i64, _int, _int, _int, _c_u64, _vp,
                             ctypes.c_float, _vp, _vp]),
    "rrq_qk_scores_qjl": (_int, [_vp, _int, _vp, _vp, _vp, _vp, _vp, _c_i64, _int, _int, _int,
                                 _c_u64, _vp, ctypes.c_float, _vp, _vp]),
    "rrq_attention_decode": (_int, [_vp, _int, _vp, _vp, _vp, _vp, _c_i64, _int, _int, _int,
                                    _c_u64, _vp, _int, _c_u64, _vp, ctypes.c_float, _vp,
                                    ctypes.c_size_t, _vp, _vp]),
    "rrq_attention_workspace_bytes": (ctypes.c_size_t, [_int, _int, _int, _int, _int, _c_i64]),
    "rrq_attention_decode_noalloc": (_int, [_vp, _int, _vp, _vp, _vp, _vp, _c_i64, _int, _int,
                                            _int, _c_u64, _vp, _int, _c_u64, _vp, ctypes.c_float,
                                            _vp, _vp]),
    "rrq_q4_0_rot": (_int, [_vp, _int, _c_i64, _int, _c_u64, _int, _vp, _vp]),
    "rrq_q4_0_rot_decode": (_int, [_vp, _c_i64, _int, _c_u64, _int, _vp, _int, _vp]),
    "rrq_ggml_block_bytes": (_int, [_int]),
    "rrq_ggml_rot": (_int, [_vp, _int, _c_i64, _int, _c_u64, _int, _int, _vp, _vp]),
    "rrq_ggml_rot_decode": (_int, [_vp, _int, _c_i64, _int, _c_u64, _int, _vp, _int, _vp]),
    "rrq_qjl_matrix": (_int, [_c_u64, _int, _vp]),
}


class RRQError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {strerror(status)} (status {status})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m random_rotation_kv_b200.build` "
                "(there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


def strerror(status: int) -> str:
    return lib().rrq_strerror(status).decode()


def _check(status: int, what: str) -> None:
    if status != RRQ_OK:
        raise RRQError(status, what)


def _dev_tensor(t: torch.Tensor, name: str, dtypes=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")


def _stream(t: torch.Tensor) -> _vp:
    return _vp(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t) -> _vp:
    return _vp(None) if t is None else _vp(t.data_ptr())


class _HostFloats:
    """Keeps a host float32 copy of a codebook alive for the duration of a call."""

    def __init__(self, codebook):
        self.arr = None if codebook is None else np.ascontiguousarray(
            np.asarray(codebook, dtype=np.float32))

    @property
    def ptr(self) -> _vp:
        return _vp(None) if self.arr is None else _vp(self.arr.ctypes.data)


def rrq_format_version() -> int:
    return lib().rrq_format_version()


def rrq_codebook(bits: int) -> np.ndarray:
    """Default codebook: ascending Lloyd–Max levels for N(0,1), float32[2^bits]."""
    out = np.zeros(1 << bits if 1 <= bits <= 8 else 1, dtype=np.float32)
    _check(lib().rrq_codebook(bits, _vp(out.ctypes.data)), "rrq_codebook")
    return out


def rrq_rotate(x: torch.Tensor, seed: int, inverse: bool = False, out: torch.Tensor | None = None):
    """Πx (or Πᵀx) of every row of x [..., d]; float32 result of x's shape."""
    _dev_tensor(x, "x", DTYPE_CODE)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    if out is None:
        out = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    _dev_tensor(out, "out", (torch.float32,))
    _check(lib().rrq_rotate(_ptr(x), DTYPE_CODE[x.dtype], n, d, seed, int(bool(inverse)),
                            _ptr(out), _stream(x)), "rrq_rotate")
    return out


def rrq_encode(x: torch.Tensor, bits: int, seed: int, codebook=None, codes=None, norms=None,
               qjl_S=None, qjl_bits=None, qjl_rnorm=None):
    """Encode rows of x [..., d].

    Returns (codes uint8 [..., d*bits/8], norms float32 [...]) and, with
    ``qjl_S`` (bf16 [d, d] on the device), also (qjl_bits uint8 [..., d/8],
    qjl_rnorm float32 [...]).
    """
    _dev_tensor(x, "x", DTYPE_CODE)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    lead = x.shape[:-1]
    if codes is None:
        codes = torch.empty(*lead, d * bits // 8, dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty(lead, dtype=torch.float32, device=x.device)
    _dev_tensor(codes, "codes", (torch.uint8,))
    _dev_tensor(norms, "norms", (torch.float32,))
    if codes.numel() != n * (d * bits // 8) or norms.numel() != n:
        raise ValueError("codes / norms have the wrong size")
    if qjl_S is not None:
        _dev_tensor(qjl_S, "qjl_S", (torch.bfloat16,))
        if qjl_S.shape != (d, d):
            raise ValueError("qjl_S must be [d, d]")
        if qjl_bits is None:
            qjl_bits = torch.empty(*lead, d // 8, dtype=torch.uint8, device=x.device)
        if qjl_rnorm is None:
            qjl_rnorm = torch.empty(lead, dtype=torch.float32, device=x.device)
        _dev_tensor(qjl_bits, "qjl_bits", (torch.uint8,))
        _dev_tensor(qjl_rnorm, "qjl_rnorm", (torch.float32,))
    cb = _HostFloats(codebook)
    _check(lib().rrq_encode(_ptr(x), DTYPE_CODE[x.dtype], n, d, bits, seed, cb.ptr, _ptr(codes),
                            _ptr(norms), _ptr(qjl_S), _ptr(qjl_bits), _ptr(qjl_rnorm),
                            _stream(x)), "rrq_encode")
    if qjl_S is not None:
        return codes, norms, qjl_bits, qjl_rnorm
    return codes, norms


def rrq_drive_encode(x: torch.Tensor, seed: int, unbiased: bool, codes=None, scales=None):
    """DRIVE one-bit encode of rows of x [..., d].

    Returns (codes uint8 [..., d/8], scales float32 [...]); scales hold S·√d,
    which rrq_decode / rrq_qk_scores with bits=1 and codebook [-1, 1] read as
    the norm.
    """
    _dev_tensor(x, "x", DTYPE_CODE)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    lead = x.shape[:-1]
    if codes is None:
        codes = torch.empty(*lead, d // 8, dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(lead, dtype=torch.float32, device=x.device)
    _dev_tensor(codes, "codes", (torch.uint8,))
    _dev_tensor(scales, "scales", (torch.float32,))
    if codes.numel() != n * (d // 8) or scales.numel() != n:
        raise ValueError("codes / scales have the wrong size")
    _check(lib().rrq_drive_encode(_ptr(x), DTYPE_CODE[x.dtype], n, d, seed, int(bool(unbiased)),
                                  _ptr(codes), _ptr(scales), _stream(x)), "rrq_drive_encode")
    return codes, scales


def rrq_decode(codes: torch.Tensor, norms: torch.Tensor, d: int, bits: int, seed: int,
               codebook=None, out_dtype=torch.float16, out=None):
    """Reconstruct vectors [..., d] of ``out_dtype`` from codes [..., d*bits/8] and norms [...]."""
    _dev_tensor(codes, "codes", (torch.uint8,))
    _dev_tensor(norms, "norms", (torch.float32,))
    n = norms.numel()
    if codes.numel() != n * (d * bits // 8):
        raise ValueError("codes / norms sizes disagree")
    if out is None:
        out = torch.empty(*norms.shape, d, dtype=out_dtype, device=codes.device)
    _dev_tensor(out, "out", DTYPE_CODE)
    if out.numel() != n * d:
        raise ValueError("out has the wrong size")
    cb = _HostFloats(codebook)
    _check(lib().rrq_decode(_ptr(codes), _ptr(norms), n, d, bits, seed, cb.ptr, _ptr(out),
                            DTYPE_CODE[out.dtype], _stream(codes)), "rrq_decode")
    return out


def rrq_qk_scores(q: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor, hkv: int, d: int,
                  bits: int, seed: int, codebook=None, scale: float = 1.0, out=None):
    """Scores [hq, T] of unrotated fp16 queries q [hq, d] against a quantised K cache.

    codes: [T*hkv, d*bits/8] (row t*hkv + g) or [T, hkv, d*bits/8]; norms: T*hkv floats.
    """
    _dev_tensor(q, "q", (torch.float16,))
    _dev_tensor(codes, "codes", (torch.uint8,))
    _dev_tensor(norms, "norms", (torch.float32,))
    hq = q.shape[0]
    if q.shape != (hq, d):
        raise ValueError("q must be [hq, d]")
    rows = norms.numel()
    if rows % hkv:
        raise ValueError("norms must hold T*hkv values")
    t_len = rows // hkv
    if codes.numel() != rows * (d * bits // 8):
        raise ValueError("codes / norms sizes disagree")
    if out is None:
        out = torch.empty(hq, t_len, dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", (torch.float32,))
    cb = _HostFloats(codebook)
    _check(lib().rrq_qk_scores(_ptr(q), hq, _ptr(codes), _ptr(norms), t_len, hkv, d, bits, seed,
                               cb.ptr, float(scale), _ptr(out), _stream(q)), "rrq_qk_scores")
    return out


def rrq_qk_scores_qjl(q: torch.Tensor, codes: torch.Tensor, norms: torch.Tensor,
                      qjl_bits: torch.Tensor, qjl_rnorm: torch.Tensor, qjl_S: torch.Tensor, hkv: int,
                      d: int, bits: int, seed: int, codebook=None, scale: float = 1.0, out=None):
    """Unbiased scores [hq, T] of unrotated fp16 queries q [hq, d] against keys stored as
    b-bit codes + norms plus the QJL sign bits and residual norms (rows t*hkv + g), with
    the projection qjl_S (bf16 [d, d]) they were encoded with."""
    _dev_tensor(q, "q", (torch.float16,))
    _dev_tensor(codes, "codes", (torch.uint8,))
    _dev_tensor(norms, "norms", (torch.float32,))
    _dev_tensor(qjl_bits, "qjl_bits", (torch.uint8,))
    _dev_tensor(qjl_rnorm, "qjl_rnorm", (torch.float32,))
    _dev_tensor(qjl_S, "qjl_S", (torch.bfloat16,))
    hq = q.shape[0]
    if q.shape != (hq, d) or qjl_S.shape != (d, d):
        raise ValueError("q must be [hq, d] and qjl_S [d, d]")
    rows = norms.numel()
    if rows % hkv:
        raise ValueError("norms must hold T*hkv values")
    t_len = rows // hkv
    if (codes.numel() != rows * (d * bits // 8) or qjl_bits.numel() != rows * (d // 8)
            or qjl_rnorm.numel() != rows):
        raise ValueError("codes / norms / qjl sizes disagree")
    if out is None:
        out = torch.empty(hq, t_len, dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", (torch.float32,))
    cb = _HostFloats(codebook)
    _check(lib().rrq_qk_scores_qjl(_ptr(q), hq, _ptr(codes), _ptr(norms), _ptr(qjl_bits),
                                   _ptr(qjl_rnorm), _ptr(qjl_S), t_len, hkv, d, bits, seed, cb.ptr,
                                   float(scale), _ptr(out), _stream(q)), "rrq_qk_scores_qjl")
    return out


def rrq_attention_decode(q: torch.Tensor, k_codes: torch.Tensor, k_norms: torch.Tensor,
                         v_codes: torch.Tensor, v_norms: torch.Tensor, hkv: int, d: int,
                         k_seed: int, v_seed: int, k_bits: int = 4, v_bits: int = 4,
                         k_codebook=None, v_codebook=None, scale: float = 1.0, out=None,
                         workspace=None):
    """One decode step of attention, out [hq, d] float32, of unrotated fp16 queries q [hq, d]
    over a K/V cache of k_bits / v_bits codes + norms (rows t*hkv + g).

    ``workspace``: a uint8 device tensor of at least rrq_attention_workspace_bytes(...)
    bytes, zero before its first use (each call leaves it ready for the next); a zeroed
    one is allocated when none is given."""
    _dev_tensor(q, "q", (torch.float16,))
    for t_, nm in ((k_codes, "k_codes"), (v_codes, "v_codes")):
        _dev_tensor(t_, nm, (torch.uint8,))
    for t_, nm in ((k_norms, "k_norms"), (v_norms, "v_norms")):
        _dev_tensor(t_, nm, (torch.float32,))
    hq = q.shape[0]
    if q.shape != (hq, d):
        raise ValueError("q must be [hq, d]")
    rows = k_norms.numel()
    if rows % hkv or v_norms.numel() != rows:
        raise ValueError("norms must hold T*hkv values")
    t_len = rows // hkv
    if k_codes.numel() != rows * (d * k_bits // 8) or v_codes.numel() != rows * (d * v_bits // 8):
        raise ValueError("codes / norms sizes disagree")
    if out is None:
        out = torch.empty(hq, d, dtype=torch.float32, device=q.device)
    _dev_tensor(out, "out", (torch.float32,))
    need = rrq_attention_workspace_bytes(hq, hkv, d, t_len, k_bits, v_bits)
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=q.device)
    _dev_tensor(workspace, "workspace", (torch.uint8,))
    kc, vc = _HostFloats(k_codebook), _HostFloats(v_codebook)
    _check(lib().rrq_attention_decode(_ptr(q), hq, _ptr(k_codes), _ptr(k_norms), _ptr(v_codes),
                                      _ptr(v_norms), t_len, hkv, d, k_bits, k_seed, kc.ptr, v_bits,
                                      v_seed, vc.ptr, float(scale), _ptr(workspace),
                                      workspace.numel(), _ptr(out), _stream(q)),
           "rrq_attention_decode")
    return out


def rrq_attention_workspace_bytes(hq: int, hkv: int, d: int, t_len: int, k_bits: int = 4,
                                  v_bits: int = 4) -> int:
    """Workspace bytes rrq_attention_decode needs on the current device."""
    return int(lib().rrq_attention_workspace_bytes(hq, hkv, d, k_bits, v_bits, t_len))


def rrq_q4_0_rot(x: torch.Tensor, seed: int, rotate: bool = True, out=None):
    """Rotate (optionally) and q4_0-quantise rows of x [..., d] -> uint8 [..., d/32*18]."""
    _dev_tensor(x, "x", DTYPE_CODE)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    if out is None:
        out = torch.empty(*x.shape[:-1], d // 32 * 18, dtype=torch.uint8, device=x.device)
    _dev_tensor(out, "out", (torch.uint8,))
    if out.numel() != n * (d // 32 * 18):
        raise ValueError("out has the wrong size")
    _check(lib().rrq_q4_0_rot(_ptr(x), DTYPE_CODE[x.dtype], n, d, seed, int(bool(rotate)),
                              _ptr(out), _stream(x)), "rrq_q4_0_rot")
    return out


def rrq_q4_0_rot_decode(blocks: torch.Tensor, d: int, seed: int, rotate: bool = True,
                        out_dtype=torch.float16, out=None):
    _dev_tensor(blocks, "blocks", (torch.uint8,))
    per = d // 32 * 18
    if blocks.shape[-1] != per:
        raise ValueError("blocks must be [..., d/32*18]")
    n = blocks.numel() // per
    if out is None:
        out = torch.empty(*blocks.shape[:-1], d, dtype=out_dtype, device=blocks.device)
    _dev_tensor(out, "out", DTYPE_CODE)
    _check(lib().rrq_q4_0_rot_decode(_ptr(blocks), n, d, seed, int(bool(rotate)), _ptr(out),
                                     DTYPE_CODE[out.dtype], _stream(blocks)),
           "rrq_q4_0_rot_decode")
    return out


def rrq_ggml_block_bytes(fmt: str) -> int:
    """Bytes of one block of 32 values of a GGML block type ('q4_0', 'q4_1', 'q5_0', 'q5_1', 'q8_0')."""
    return lib().rrq_ggml_block_bytes(GGML_TYPES[fmt])


def rrq_ggml_rot(x: torch.Tensor, seed: int, fmt: str, rotate: bool = True, out=None):
    """Rotate (optionally) then quantise rows of x [..., d] into GGML blocks of type `fmt`:
    uint8 [..., d/32*block_bytes]."""
    _dev_tensor(x, "x", DTYPE_CODE)
    d = x.shape[-1]
    n = x.numel() // d if d else 0
    per = d // 32 * rrq_ggml_block_bytes(fmt)
    if out is None:
        out = torch.empty(*x.shape[:-1], per, dtype=torch.uint8, device=x.device)
    _dev_tensor(out, "out", (torch.uint8,))
    if out.numel() != n * per:
        raise ValueError("out has the wrong size")
    _check(lib().rrq_ggml_rot(_ptr(x), DTYPE_CODE[x.dtype], n, d, seed, int(bool(rotate)),
                              GGML_TYPES[fmt], _ptr(out), _stream(x)), "rrq_ggml_rot")
    return out


def rrq_ggml_rot_decode(blocks: torch.Tensor, d: int, seed: int, fmt: str, rotate: bool = True,
                        out_dtype=torch.float16, out=None):
    _dev_tensor(blocks, "blocks", (torch.uint8,))
    per = d // 32 * rrq_ggml_block_bytes(fmt)
    if blocks.shape[-1] != per:
        raise ValueError(f"blocks must be [..., d/32*{per // (d // 32)}]")
    n = blocks.numel() // per
    if out is None:
        out = torch.empty(*blocks.shape[:-1], d, dtype=out_dtype, device=blocks.device)
    _dev_tensor(out, "out", DTYPE_CODE)
    _check(lib().rrq_ggml_rot_decode(_ptr(blocks), GGML_TYPES[fmt], n, d, seed, int(bool(rotate)),
                                     _ptr(out), DTYPE_CODE[out.dtype], _stream(blocks)),
           "rrq_ggml_rot_decode")
    return out


def rrq_qjl_matrix(seed: int, d: int, device=None) -> torch.Tensor:
    """The QJL projection S (bf16 [d, d]); generated on the host by the library, then copied."""
    host = np.zeros(d * d if d > 0 else 1, dtype=np.uint16)
    _check(lib().rrq_qjl_matrix(seed, d, _vp(host.ctypes.data)), "rrq_qjl_matrix")
    t = torch.from_numpy(host.view(np.int16).copy()).view(torch.bfloat16).reshape(d, d)
    return t if device is None else t.to(device)
