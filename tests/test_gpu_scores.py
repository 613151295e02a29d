"""GPU-vs-oracle parity for rrq_qk_scores (attention scores on packed codes; needs a B200).

The GPU scores the oracle's own codes and norms, so the comparison isolates the
score kernel: |s_gpu − s_oracle| ≤ 1e-3·‖q‖·‖k̂‖·|scale| for every (head, token).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import rrq as orc
from random_rotation_kv_b200 import binding as B
from random_rotation_kv_b200 import workloads as W
from tests import parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(t_len, hkv, hq, d, bits, seed=42, scale=1.0, data_seed=0, codebook=None):
    rng = np.random.default_rng(data_seed + 1000 * bits + d)
    k = W.kv(tokens=t_len, heads=hkv, d=d, bits=bits, seed=1005 + data_seed).flat()
    q = rng.standard_normal((hq, d)).astype(np.float16)
    levels = None if codebook is None else np.asarray(codebook, np.float64)
    enc = orc.encode(k.astype(np.float64), bits, seed, levels)
    s_gpu = B.rrq_qk_scores(torch.from_numpy(q).to(DEV), torch.from_numpy(enc.packed).to(DEV),
                            torch.from_numpy(enc.norms).to(DEV), hkv, d, bits, seed,
                            codebook=codebook, scale=scale)
    torch.cuda.synchronize()
    s_orc = orc.scores(q.astype(np.float64), enc.packed, enc.norms, t_len, hkv, d, bits, seed,
                       levels, scale)
    cs = orc.score_tolerance_scale(q.astype(np.float64), enc.packed, enc.norms, t_len, hkv, d,
                                   bits, levels)
    P.assert_scores_close(s_gpu.cpu().numpy(), s_orc, cs, scale,
                          f"scores T={t_len} hkv={hkv} hq={hq} d={d} b={bits}")
    return s_gpu


@pytest.mark.parametrize("d", [64, 128, 256, 512])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_scores_parity_sweep(d, bits):
    _case(301, 8, 32, d, bits)


@pytest.mark.parametrize("hq,hkv", [(8, 8), (8, 1), (16, 2), (32, 4), (64, 8), (4, 4), (32, 16)])
def test_scores_gqa_layouts(hq, hkv):
    _case(257, hkv, hq, 128, 4, data_seed=hq + hkv)


@pytest.mark.parametrize("d,hkv", [(512, 8), (256, 16), (512, 16), (64, 1), (64, 32)])
def test_scores_head_blocks_and_token_groups(d, hkv):
    _case(133, hkv, hkv * 2, d, 4, data_seed=d + hkv)


@pytest.mark.parametrize("t_len", [1, 2, 127, 128, 129, 1000])
def test_scores_ragged_token_counts(t_len):
    _case(t_len, 8, 32, 128, 4, data_seed=t_len)


def test_scores_scale_and_custom_codebook():
    cb = np.sort(np.random.default_rng(5).normal(size=16)).astype(np.float32)
    _case(200, 8, 32, 128, 4, scale=1 / math.sqrt(128), codebook=cb)


def test_scores_zero_query_head():
    hq, hkv, d, t_len = 8, 8, 128, 64
    k = W.kv(tokens=t_len, heads=hkv).flat()
    enc = orc.encode(k.astype(np.float64), 4, 42)
    q = np.zeros((hq, d), np.float16)
    s = B.rrq_qk_scores(torch.from_numpy(q).to(DEV), torch.from_numpy(enc.packed).to(DEV),
                        torch.from_numpy(enc.norms).to(DEV), hkv, d, 4, 42)
    torch.cuda.synchronize()
    assert torch.all(s == 0)


def test_scores_full_size_sampled():
    """The benchmarked shape: 131072 tokens x 8 KV heads, 32 query heads, d = 128, b = 4."""
    w = W.scores()
    k = torch.from_numpy(w.flat()).to(DEV)
    codes, norms = B.rrq_encode(k, 4, 42)
    q = w.extra["q"]
    s = B.rrq_qk_scores(torch.from_numpy(q).to(DEV), codes, norms, 8, 128, 4, 42)
    torch.cuda.synchronize()
    t_len = w.x.shape[0]
    toks = np.sort(np.random.default_rng(1).choice(t_len, 2000, replace=False))
    toks = np.concatenate([toks, [0, t_len - 1]])
    rows = (toks[:, None] * 8 + np.arange(8)[None, :]).ravel()
    pk = codes[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    nk = norms[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    s_orc = orc.scores(q.astype(np.float64), pk, nk, len(toks), 8, 128, 4, 42)
    cs = orc.score_tolerance_scale(q.astype(np.float64), pk, nk, len(toks), 8, 128, 4)
    P.assert_scores_close(s[:, torch.from_numpy(toks).to(DEV)].cpu().numpy(), s_orc, cs, 1.0,
                          "full-size scores")


def test_scores_unsupported_layouts_raise():
    q = torch.zeros(12, 128, dtype=torch.float16, device=DEV)
    codes = torch.zeros(16 * 6, 64, dtype=torch.uint8, device=DEV)
    norms = torch.zeros(16 * 6, dtype=torch.float32, device=DEV)
    with pytest.raises(B.RRQError) as e:
        B.rrq_qk_scores(q, codes, norms, 6, 128, 4, 42)  # hkv not a power of two
    assert e.value.status == B.RRQ_ERR_UNSUPPORTED
