"""Host-side multi-rank logic of bench.py on CPU: world-size-2 gloo ranks.

Every rank encodes its own batch (weak scaling, no collective on the data path).
The only collective is a MAX all-reduce of the timed milliseconds, and the job's
throughput is the units all ranks processed over that slowest time.
"""

from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        local_ms = [12.5, 40.0][rank]
        mx = bench.max_over_ranks(local_ms, world, "cpu")
        e2e = bench.max_over_ranks(float(rank + 1), world, "cpu")
        val = bench.job_throughput(world, bench.N_VEC, 10, mx)
        out.put((rank, mx, e2e, val, bench.rank_seed(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_units():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, e2e, val, seed in res:
        assert mx == 40.0 and e2e == 2.0  # every rank sees the slowest rank's time
        assert val == pytest.approx(2 * bench.N_VEC * 10 / 0.040)
    assert res[0][4] != res[1][4]  # each rank has its own batch


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_throughput(1, 100, 4, 2.0) == pytest.approx(200000.0)


def test_rank_batches_differ():
    from random_rotation_kv_b200 import workloads as W
    a = W.kv(tokens=8, seed=bench.rank_seed(0)).flat()
    b = W.kv(tokens=8, seed=bench.rank_seed(1)).flat()
    assert a.shape == b.shape and not np.array_equal(a, b)


def test_reference_arm_runs_on_rank0_only(capsys, monkeypatch):
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup, gpus, ref_budget, ref_sample = 3, 3, 2, 1.0, 64
    bench.run_reference(Args())
    assert capsys.readouterr().out == ""
