"""Host logic of the KV encoder's code search, on the CPU (no GPU needed).

The encoders for d = 128 at 4 bits and the QJL kernel decide a coordinate's code
from its fixed-point value I = round(u·2^18) (u = y'/ν) in one integer add: the
host builds, per cell j = ⌊I / 2^16⌋ + 64 (a quarter of a unit of u), an offset
off_j such that byte 2 of 0x4B400000 + I + off_j is #{k : I > T_k}, with
T_k = ⌊τ_k·2^18⌋ and τ_k the midpoints of the codebook ("Random-rotation
quantization" page, scheme step 2: the nearest level of a fixed Lloyd–Max
codebook).  This test compiles the host function with nvcc, asks it for the
tables of several codebooks, and checks every table against the counting rule
written out here, on every I near a threshold and on random I over the whole
reachable range |I| < 2^22; a codebook with two thresholds in one reachable cell
must be refused.
"""

from __future__ import annotations

import os
import shutil
import subprocess

import numpy as np
import pytest

from oracle import codebook as ocb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "random_rotation_kv_b200", "csrc")

PROG = r"""
#include <cstdio>
#include "batch_kernels.cuh"  // the encoders' headers, mma_encode.cuh among them
int main() {
  int bits = 0;
  if (std::scanf("%d", &bits) != 1) return 2;
  rrq::QuantParams p{};
  p.bits = bits;
  for (int k = 0; k < (1 << bits); ++k) {
    double v = 0;
    if (std::scanf("%lf", &v) != 1) return 2;
    p.levels[k] = float(v);
  }
  const rrq::FixedSearch fs = rrq::make_fixed_search(p);
  std::printf("%d\n", fs.ok);
  for (int r = 0; r < 128; ++r) std::printf("%u\n", fs.off[r]);
  return 0;
}
"""


@pytest.fixture(scope="module")
def table_tool(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("fixed_search")
    src, exe = d / "tool.cu", d / "tool"
    src.write_text(PROG)
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, str(src), "-o", str(exe), "-lcudart"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    return str(exe)


def tables(tool, levels):
    levels = np.asarray(levels, np.float32)
    bits = int(np.log2(levels.size))
    inp = f"{bits} " + " ".join(repr(float(v)) for v in levels)
    res = subprocess.run([tool], input=inp, capture_output=True, text=True, check=True)
    vals = [int(v) for v in res.stdout.split()]
    return vals[0], np.array(vals[1:], dtype=np.int64)


def thresholds_fixed(levels):
    lv = np.asarray(levels, np.float32).astype(np.float64)
    tau = (lv[:-1] + lv[1:]) * 0.5
    return np.clip(np.floor(tau * 262144.0), -8388608, 8388608).astype(np.int64)


def check_table(off, T, rng):
    near = np.concatenate([T + dlt for dlt in (-2, -1, 0, 1, 2)])
    I = np.concatenate([near, rng.integers(-(1 << 22), 1 << 22, 300000)])
    I = I[(I >= -(1 << 22)) & (I < (1 << 22))]
    f = (0x4B400000 + I) % (1 << 32)
    cell = (f >> 16) & 0xFF
    assert cell.min() >= 0 and cell.max() < 128
    code = (((f + off[cell]) % (1 << 32)) >> 16) & 0xFF
    want = (I[:, None] > T[None, :]).sum(axis=1)
    bad = np.flatnonzero(code != want)
    assert bad.size == 0, f"I = {I[bad[:5]]}: table gives {code[bad[:5]]}, rule {want[bad[:5]]}"


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_default_codebooks(table_tool, bits):
    lv = ocb.lloyd_max(bits)
    ok, off = tables(table_tool, lv)
    assert ok == 1
    check_table(off, thresholds_fixed(lv), np.random.default_rng(bits))


@pytest.mark.parametrize("scale", [1e-3, 0.5, 7.0, 40.0])
def test_scaled_and_asymmetric_codebooks(table_tool, scale):
    """Narrow and wide codebooks (thresholds far outside the reachable |u| ≤ √128 are
    clamped and never change a decision) and an asymmetric one."""
    for lv in (ocb.lloyd_max(4) * scale, np.array([-2.0, -0.7, -0.1, 0.4, 0.9, 1.3, 2.2, 3.5]) * scale):
        ok, off = tables(table_tool, lv)
        T = thresholds_fixed(lv)
        reach = T[(T >= -(64 << 16)) & (T < (64 << 16))]
        if np.any(np.diff(reach >> 16) == 0):
            assert ok == 0  # two thresholds in one reachable cell: refused
        else:
            assert ok == 1
            check_table(off, T, np.random.default_rng(int(scale * 1000)))


def test_two_thresholds_in_one_cell_are_refused(table_tool):
    ok, _ = tables(table_tool, [-1.0, -0.95, -0.9, 1.0])  # midpoints 0.05 apart
    assert ok == 0
