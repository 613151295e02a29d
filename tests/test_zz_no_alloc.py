"""The allocation-free attention entry point, rrq_attention_decode_noalloc (needs a B200).

Some callers cannot allocate device memory where they call the library (a serving
loop whose memory an allocator of its own reserved up front, or code with no
workspace to hand down); this entry point runs the attention kernel with its
scratch in a fixed 4 MiB array inside the library.  The test calls it through the
C ABI twice in a row, on the same inputs, and compares each output with the
workspace entry point's within the attention tolerance of test_gpu_attention.py
(per head, 2e-3 of the softmax-weighted sum of the value reconstruction norms,
with the weights from the oracle); it also checks that a request
larger than the array is refused before anything runs.  This file is collected
last, so that a run stopping at its first failure has run every other test.
"""

from __future__ import annotations

import ctypes
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from random_rotation_kv_b200 import binding as B
from tests.parity import attention_bound as weighted_bound

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
D = 128


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(q, kc, kn, vc, vn, hkv, out, scale, d=D, kb=4, vb=4):
    hq = q.shape[0]
    t_len = kn.numel() // hkv
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return B.lib().rrq_attention_decode_noalloc(
        _ptr(q), hq, _ptr(kc), _ptr(kn), _ptr(vc), _ptr(vn), t_len, hkv, d, kb, 42, None, vb, 43,
        None, ctypes.c_float(scale), _ptr(out), stream)


def test_noalloc_attention_matches_the_workspace_entry_twice():
    rg = np.random.Generator(np.random.PCG64(2024))
    t_len, hkv, hq = 20000, 8, 32
    rows = t_len * hkv
    kc = torch.from_numpy(rg.integers(0, 256, size=(rows, 64), dtype=np.uint8)).to(DEV)
    vc = torch.from_numpy(rg.integers(0, 256, size=(rows, 64), dtype=np.uint8)).to(DEV)
    kn = torch.from_numpy((np.exp(rg.standard_normal(rows) * 0.5) * 11.0).astype(np.float32)).to(DEV)
    vn = torch.from_numpy((np.exp(rg.standard_normal(rows) * 0.5) * 9.0).astype(np.float32)).to(DEV)
    q = torch.from_numpy(rg.standard_normal((hq, D)).astype(np.float16)).to(DEV)
    scale = 1.0 / math.sqrt(D)
    ref = B.rrq_attention_decode(q, kc, kn, vc, vn, hkv, D, 42, 43, scale=scale)
    torch.cuda.synchronize()
    host = [t.cpu().numpy() for t in (q, kc, kn, vc, vn)]
    _, p = oatt.decode_attention(*host, t_len, hkv, D, 4, 4, 42, 43, scale=scale,
                                 return_weights=True)
    bound = torch.from_numpy(weighted_bound(p, host[3], host[4], t_len, hkv, D, 4, 43)).to(DEV)
    for _ in range(2):
        out = torch.full((hq, D), float("nan"), dtype=torch.float32, device=DEV)
        assert _noalloc(q, kc, kn, vc, vn, hkv, out, scale) == B.RRQ_OK
        torch.cuda.synchronize()
        err = torch.linalg.norm((out - ref).double(), dim=1)
        assert torch.all(err <= bound), float(err.max())


def test_noalloc_attention_other_shapes_twice():
    """d = 64 with 2-bit K and 3-bit V (the scores go to the scratch array too)."""
    rg = np.random.Generator(np.random.PCG64(2025))
    t_len, hkv, hq, d = 3000, 4, 16, 64
    rows = t_len * hkv
    kc = torch.from_numpy(rg.integers(0, 256, size=(rows, d * 2 // 8), dtype=np.uint8)).to(DEV)
    vc = torch.from_numpy(rg.integers(0, 256, size=(rows, d * 3 // 8), dtype=np.uint8)).to(DEV)
    kn = torch.from_numpy((np.exp(rg.standard_normal(rows) * 0.5) * 8.0).astype(np.float32)).to(DEV)
    vn = torch.from_numpy((np.exp(rg.standard_normal(rows) * 0.5) * 6.0).astype(np.float32)).to(DEV)
    q = torch.from_numpy(rg.standard_normal((hq, d)).astype(np.float16)).to(DEV)
    assert B.rrq_attention_workspace_bytes(hq, hkv, d, t_len, 2, 3) <= 4 << 20
    host = [t.cpu().numpy() for t in (q, kc, kn, vc, vn)]
    ref, p = oatt.decode_attention(*host, t_len, hkv, d, 2, 3, 42, 43, scale=0.125, return_weights=True)
    bound = weighted_bound(p, host[3], host[4], t_len, hkv, d, 3, 43)
    for _ in range(2):
        out = torch.full((hq, d), float("nan"), dtype=torch.float32, device=DEV)
        assert _noalloc(q, kc, kn, vc, vn, hkv, out, 0.125, d, 2, 3) == B.RRQ_OK
        torch.cuda.synchronize()
        err = np.linalg.norm(out.cpu().numpy().astype(np.float64) - ref, axis=1)
        assert np.all(err <= bound), float(np.max(err / bound))


def test_noalloc_attention_refuses_requests_beyond_its_scratch():
    # 8192 query heads over 1024 kv heads (group 8) need far more than 4 MiB of partial states
    hq, hkv, t_len = 8, 1, 64
    need = B.rrq_attention_workspace_bytes(hq * 1024, hkv * 1024, D, t_len)
    assert need > 4 << 20
    kc = torch.zeros(t_len * hkv * 1024, 64, dtype=torch.uint8, device=DEV)
    kn = torch.ones(t_len * hkv * 1024, dtype=torch.float32, device=DEV)
    q = torch.zeros(hq * 1024, D, dtype=torch.float16, device=DEV)
    out = torch.full((hq * 1024, D), 7.0, dtype=torch.float32, device=DEV)
    assert _noalloc(q, kc, kn, kc, kn, hkv * 1024, out, 1.0) == B.RRQ_ERR_SCRATCH
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)  # nothing ran
