#!/usr/bin/env python
"""Benchmark: fp16 KV-cache vectors encoded + decoded per second on B200.

Workload (one step): the fp16 K cache [32768 tokens × 8 KV heads × 128]
(262,144 vectors; 2 % outlier channels ×15, log-normal per-token scale),
encoded at 4 bits (randomized Hadamard rotation + N(0,1) Lloyd–Max codes +
fp32 norm) and decoded back to fp16, through the C ABI (rrq_encode,
rrq_decode).  Inputs are resident in HBM before timing starts.  The timed
steps run back to back between one pair of CUDA events, over 4 rotating
batches (4 × 84.9 MB per kernel kind, larger than the 126 MB L2): step k
encodes batch k mod 4 and decodes the codes of batch (k + 2) mod 4, written two
steps earlier and evicted from L2 since.  The per-kernel figures (roofline)
come from encode-only and decode-only loops timed the same way; a flushed
single-launch figure (256 MiB write before each launch) is reported beside
them.  Multi-GPU (torchrun): every rank processes its own batches of the same
size (weak scaling, no collective on the data path); the time is the maximum
over ranks.

``--impl reference`` times the CPU oracle (the plain fp64 restatement under
``oracle/``) on a bounded sample of the same workload instead.

Prints one JSON line (rank 0).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV vectors/s encode+decode (d=128,b=4, fp16); achieved HBM GB/s vs peak"
UNIT = "vectors/s"
TOKENS, HEADS, D, BITS = 32768, 8, 128, 4
N_VEC = TOKENS * HEADS
BYTES_PER_VEC_ENC = D * 2 + D * BITS // 8 + 4   # read fp16, write codes + fp32 norm
BYTES_PER_VEC_DEC = D * BITS // 8 + 4 + D * 2   # read codes + norm, write fp16
NOMINAL_HBM_GBS = 8000.0
ROT = 4  # rotating batches: 4 x 84.9 MB per kernel kind, larger than the 126 MB L2
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["random_rotation_kv_b200/csrc/rrq_device.cuh",
                  "random_rotation_kv_b200/csrc/quant_kernels.cuh",
                  "random_rotation_kv_b200/csrc/batch_kernels.cuh",
                  "random_rotation_kv_b200/csrc/tc_encode.cuh",
                  "random_rotation_kv_b200/csrc/tcgen05.cuh",
                  "random_rotation_kv_b200/csrc/mma_encode.cuh",
                  "random_rotation_kv_b200/csrc/mma_decode.cuh",
                  "random_rotation_kv_b200/csrc/tensor_map.h",
                  "random_rotation_kv_b200/csrc/rrq_params.h"]
# the kernels the headline's two calls run on this workload (d = 128, 4-bit, fp16)
ENCODE_KERNEL, DECODE_KERNEL = "encode_tc_kernel", "decode_mma_kernel"


def workload_config(extra=None):
    cfg = {"workload": "kv-cache K fp16 [32768 tokens x 8 kv heads x 128], 4-bit RHT + Lloyd-Max, "
                       "encode+decode",
           "vectors_per_gpu": N_VEC, "d": D, "bits": BITS, "io_dtype": "f16",
           "rotation_seed": 42,
           "l2": "inputs larger than L2: 4 rotating batches; step k encodes batch k mod 4 and "
                 "decodes the codes of batch (k+2) mod 4, written two steps earlier"}
    if extra:
        cfg.update(extra)
    return cfg


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        entry = rec[kernel]
        if entry.get("source_hash") != kernel_source_hash():
            return None
        return float(entry["dram_bytes_per_launch"])
    except Exception:
        return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return self.lines

    @staticmethod
    def summarize(lines, t0, t1):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm, smax, reasons, n = [], None, set(), 0
        for t, ln in lines or []:
            if not (t0 <= t <= t1 + 0.15):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            n += 1
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": n}


def gpu_id_for(torch, dev):
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        return str(dev)


# ------------------------------------------------------------- CPU oracle
def oracle_step_time(x_sample: np.ndarray, reps: int = 1) -> float:
    """Seconds for the oracle to encode + decode x_sample (fp16 [n, 128]), best of reps."""
    from oracle import rrq as orc
    best = float("inf")
    for _ in range(reps):
        t = time.perf_counter()
        enc = orc.encode(x_sample.astype(np.float64), BITS, 42)
        orc.decode(enc.packed, enc.norms, BITS, D, 42, out_dtype="f16")
        best = min(best, time.perf_counter() - t)
    return best


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info] + [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(x_flat: np.ndarray, budget_s: float = 12.0):
    """The oracle as it stands on a bounded sample of the workload, timed twice: with
    its BLAS on every core this process may use, and pinned to one thread.  About
    budget_s seconds of wall time each."""
    from threadpoolctl import threadpool_limits
    cores = host_cores()
    out = {}
    for label, threads in (("all", cores), ("one", 1)):
        with threadpool_limits(limits=threads):
            n0 = 2048
            t0 = oracle_step_time(x_flat[:n0])
            n = int(min(x_flat.shape[0], max(n0, n0 * budget_s / max(t0, 1e-3) / 2)))
            t = oracle_step_time(x_flat[:n])
            out[label] = (n, t, min(threads, blas_threads()))
    n, t, used = out["all"]
    n1, t1, _ = out["one"]
    return {"value": n / t, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"first {n} of the {x_flat.shape[0]} workload vectors, encode+decode, "
                      f"numpy fp64 (dense rotation matrix), {t:.2f} s wall, BLAS on {used} threads",
            "cpu_model": cpu_model(), "host_cores": cores,
            "single_thread": {"value": n1 / t1, "unit": UNIT, "cores": 1,
                              "sample": f"first {n1} workload vectors, {t1:.2f} s wall, BLAS on 1 thread"}}


# ------------------------------------------------------------ reference
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return  # rank 0 alone runs the CPU reference
    from random_rotation_kv_b200 import workloads as W
    w = W.kv()
    x = w.flat()
    # size each step's sample so that warm-up + timed steps take about
    # --ref-budget seconds of CPU in total, whatever --steps is
    rate = 2048 / oracle_step_time(x[:2048])
    per_step = args.ref_budget * rate / (args.steps + args.warmup)
    n_sample = int(min(args.ref_sample, max(128, per_step)))
    for _ in range(args.warmup):
        oracle_step_time(x[:n_sample])
    times = [oracle_step_time(x[:n_sample]) for _ in range(args.steps)]
    total = sum(times)
    value = n_sample * args.steps / total
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config({"sample_vectors_per_step": n_sample,
                                   "l2": "n/a (the CPU oracle on the host cores)"}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"first {n_sample} workload vectors per step, encode+decode",
                         "cpu_model": cpu_model(), "host_cores": host_cores()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------- GPU arm
def rank_seed(rank: int) -> int:
    """Seed of a rank's own batch of the KV workload (weak scaling: a new batch per rank)."""
    return 1002 + rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest x over all ranks: one MAX all-reduce that every rank calls in turn."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: int, steps: int, max_ms: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return world * units_per_rank * steps / (max_ms / 1e3)


def run_gpu(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize(dev)

    from random_rotation_kv_b200 import binding as B
    from random_rotation_kv_b200 import workloads as W

    # ROT batches per rank, each its own seeded KV batch (weak scaling: new data per rank)
    x_host = W.kv(seed=rank_seed(rank)).flat()
    xs = [torch.from_numpy(x_host).to(dev)]
    for j in range(1, ROT):
        xs.append(torch.from_numpy(W.kv(seed=rank_seed(rank) + 1000 * j).flat()).to(dev))
    codes = [torch.empty(N_VEC, D * BITS // 8, dtype=torch.uint8, device=dev) for _ in range(ROT)]
    norms = [torch.empty(N_VEC, dtype=torch.float32, device=dev) for _ in range(ROT)]
    outs = [torch.empty(N_VEC, D, dtype=torch.float16, device=dev) for _ in range(ROT)]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def enc(j):
        B.rrq_encode(xs[j], BITS, 42, codes=codes[j], norms=norms[j])

    def dec(j, o):
        B.rrq_decode(codes[j], norms[j], D, BITS, 42, out_dtype=torch.float16, out=outs[o])

    def step(k):
        enc(k % ROT)
        dec((k + 2) % ROT, k % ROT)  # codes written two steps earlier

    for j in range(ROT):  # every batch has codes before the first decode reads them
        enc(j)
    for k in range(args.warmup):
        step(k)
    # keep the clocks in steady state before the timed region
    t_end = time.time() + args.settle_s
    k = 0
    while time.time() < t_end:
        step(k)
        k += 1
    sampler = ClockSampler(gpu_id_for(torch, dev)) if rank == 0 and not args.no_clocks else None
    if sampler:
        sampler.start()
    barrier()
    t0 = time.time()
    step_ms = time_loop(torch, stream, step, args.steps)
    barrier()
    t1 = time.time()
    clocks = ClockSampler.summarize(sampler.stop(), t0, t1) if sampler else None
    total_ms = max_over_ranks(step_ms * args.steps, world, dev)
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, N_VEC, args.steps, total_ms)
    # per-kernel average launch durations, the same way (rotating batches, back to back)
    enc_avg = max_over_ranks(time_loop(torch, stream, lambda k: enc(k % ROT), args.steps), world, dev)
    dec_avg = max_over_ranks(time_loop(torch, stream, lambda k: dec((k + 2) % ROT, k % ROT),
                                       args.steps), world, dev)
    # single launches with L2 flushed before each (carry the fixed launch + event cost)
    enc_iso = time_kernel(torch, stream, flush, lambda: enc(0), 20)
    dec_iso = time_kernel(torch, stream, flush, lambda: dec(0, 0), 20)
    x, out, codes0, norms0 = xs[0], outs[0], codes[0], norms[0]

    # end to end through the public API: pinned host -> device -> encode -> decode -> host,
    # every step copying its own input in and its result out.  Steps are pipelined
    # over three streams and two buffer sets, so that step k's device-to-host copy,
    # step k+1's kernels and step k+2's host-to-device copy overlap (PCIe carries
    # both directions at once).
    x_pin = torch.from_numpy(x_host).pin_memory()
    out_pins = [torch.empty(N_VEC, D, dtype=torch.float16).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    o_dev = [out, torch.empty_like(out)]
    c_dev = [codes0, torch.empty_like(codes0)]
    n_dev = [norms0, torch.empty_like(norms0)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = {key: [torch.cuda.Event() for _ in range(2)] for key in ("in", "run", "out")}
    issued = {key: [False, False] for key in ("run", "out")}

    def e2e_step(k):
        j = k % 2
        with torch.cuda.stream(s_in):
            if issued["run"][j]:
                s_in.wait_event(ev["run"][j])  # the kernels of step k-2 have read x_dev[j]
            x_dev[j].copy_(x_pin, non_blocking=True)
            ev["in"][j].record(s_in)
        stream.wait_event(ev["in"][j])
        if issued["out"][j]:
            stream.wait_event(ev["out"][j])  # step k-2's result has left o_dev[j]
        B.rrq_encode(x_dev[j], BITS, 42, codes=c_dev[j], norms=n_dev[j])
        B.rrq_decode(c_dev[j], n_dev[j], D, BITS, 42, out_dtype=torch.float16, out=o_dev[j])
        ev["run"][j].record(stream)
        issued["run"][j] = True
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["run"][j])
            out_pins[j].copy_(o_dev[j], non_blocking=True)
            ev["out"][j].record(s_out)
        issued["out"][j] = True

    for k in range(3):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(args.e2e_steps):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = job_throughput(world, N_VEC, args.e2e_steps, e2e_ms)
    last = (args.e2e_steps - 1) % 2
    assert torch.equal(out_pins[last], o_dev[last].cpu())

    if rank == 0:
        peak, peak_kind = peaks()
        dom, dom_ms, dom_bytes = ((ENCODE_KERNEL, enc_avg, BYTES_PER_VEC_ENC) if enc_avg >= dec_avg
                                  else (DECODE_KERNEL, dec_avg, BYTES_PER_VEC_DEC))
        achieved = dom_bytes * N_VEC / (dom_ms / 1e3) / 1e9
        traffic = recorded_traffic(dom)
        step_gbs = (BYTES_PER_VEC_ENC + BYTES_PER_VEC_DEC) * N_VEC / (ms_per_step / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": workload_config({"parallelism": f"dp{world} (independent batches)"}),
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved,
                         "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "peak_source": f"{peak_kind} copy bandwidth",
                         "traffic": traffic,
                         "algorithmic_bytes_per_launch": dom_bytes * N_VEC},
            "hbm": {"encode_us": 1e3 * enc_avg, "decode_us": 1e3 * dec_avg,
                    "isolated_flushed_encode_us": 1e3 * enc_iso,
                    "isolated_flushed_decode_us": 1e3 * dec_iso,
                    "encode_gbs": BYTES_PER_VEC_ENC * N_VEC / (enc_avg / 1e3) / 1e9,
                    "decode_gbs": BYTES_PER_VEC_DEC * N_VEC / (dec_avg / 1e3) / 1e9,
                    "step_gbs": step_gbs, "step_frac_of_measured": step_gbs / peak,
                    "step_frac_of_nominal_8tbs": step_gbs / NOMINAL_HBM_GBS},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": N_VEC * D * 2,
                    "d2h_bytes_per_step": N_VEC * D * 2},
            "gpu_launches": 2 * args.steps,
            "clocks": clocks,
        }
        if world == 1 and not args.no_extras:
            sel = set(args.extras.split(",")) if args.extras else None
            line["kernels"] = extra_kernels(torch, dev, flush, 50, peak, sel)
            if sel is None or "reports" in sel:
                c_r, n_r = B.rrq_encode(xs[0], BITS, 42)
                x_r = B.rrq_decode(c_r, n_r, D, BITS, 42, out_dtype=torch.float32)
                kv_err = float(((x_r.double() - xs[0].double()) ** 2).sum())
                line["reports"] = {
                    "pr1": quality_reports(torch, dev),
                    "kv_headline": {"nmse": kv_err / float((xs[0].double() ** 2).sum()),
                                    "lloyd_max_distortion_D_b": lloyd_max_distortion(
                                        B.rrq_codebook(BITS))},
                    "attnrot_q4_0": {k: line["kernels"]["q4_0_rot"][k] for k in (
                        "mse_rotated", "mse_unrotated", "mse_rotated_over_unrotated")}
                    if "q4_0_rot" in line["kernels"] else None}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(x_host)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def time_loop(torch, stream, fn, steps):
    """Average device time (ms) of fn(k), k = 0..steps-1, run back to back between
    one pair of CUDA events on `stream`, after 3 untimed calls."""
    for k in range(3):
        fn(k)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for k in range(steps):
        fn(k)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def time_kernel(torch, stream, flush, fn, reps):
    """Average device time (ms) of fn() with L2 flushed (untimed) before each call."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for _ in range(3):
        flush.fill_(3)
        fn()
    for e0, e1 in evs:
        flush.fill_(4)
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    return sum(e0.elapsed_time(e1) for e0, e1 in evs) / reps


def lloyd_max_distortion(levels) -> float:
    """E[(X − Q(X))²] for X ~ N(0,1) under nearest-level quantisation with `levels`
    (ascending), summed in closed form over the cells between midpoints."""
    import math
    lv = [float(c) for c in levels]
    edges = [-math.inf] + [(lv[i] + lv[i + 1]) / 2 for i in range(len(lv) - 1)] + [math.inf]

    def phi(x):
        return 0.0 if math.isinf(x) else math.exp(-x * x / 2) / math.sqrt(2 * math.pi)

    def cdf(x):
        return 0.5 * (1 + math.erf(x / math.sqrt(2))) if not math.isinf(x) else (0.0 if x < 0 else 1.0)

    def xphi(x):
        return 0.0 if math.isinf(x) else x * phi(x)

    tot = 0.0
    for c, a, b in zip(lv, edges[:-1], edges[1:]):
        mass = cdf(b) - cdf(a)
        tot += mass * (1 + c * c) - (xphi(b) - xphi(a)) - 2 * c * (phi(a) - phi(b))
    return tot


def quality_reports(torch, dev):
    """Reconstruction error of the GPU path on the PR1 workload (4096 fp32 vectors,
    d = 128, three outlier channels x20, b = 2): MSE per coordinate, NMSE against the
    Lloyd-Max distortion D_2 of N(0,1), and the NMSE of the same codebook applied
    without the rotation.  The unrotated figure runs on the same kernels: encoding
    Πᵀx with the rotating encoder quantises the coordinates of x itself (Π·Πᵀx = x),
    and the decoder's Πᵀ is an isometry, so ‖decode − Πᵀx‖ is the unrotated error."""
    from random_rotation_kv_b200 import binding as B
    from random_rotation_kv_b200 import workloads as W
    w = W.pr1()
    x = torch.from_numpy(w.flat()).to(dev)
    d, bits = w.d, w.bits

    def nmse_of(v):
        codes, norms = B.rrq_encode(v, bits, 42)
        vh = B.rrq_decode(codes, norms, d, bits, 42, out_dtype=torch.float32)
        err = float(((vh.double() - v.double()) ** 2).sum())
        return err, err / float((v.double() ** 2).sum())

    err, nmse = nmse_of(x)
    _, nmse_u = nmse_of(B.rrq_rotate(x, 42, inverse=True))
    d_b = lloyd_max_distortion(B.rrq_codebook(bits))
    return {"workload": "PR1: 4096 fp32 vectors d=128, N(0,1) with channels {3,47,111} x20, b=2",
            "mse": err / x.numel(), "nmse": nmse, "lloyd_max_distortion_D_b": d_b,
            "nmse_over_D_b": nmse / d_b, "unrotated_nmse": nmse_u,
            "unrotated_over_rotated_nmse": nmse_u / nmse}


def scores_sweep(torch, dev, reps, peak):
    """rrq_qk_scores over d in {64, 128, 256, 512} x b in {1, 2, 3, 4}: 32 query heads
    against 131072 tokens x 8 kv heads, keys with the KV-cache distribution.  Each
    case rotates over enough copies of its cache to exceed L2 (at least 3, and at
    least 384 MB in all).  Bytes per key-head: d·b/8 code bytes + 4 norm bytes
    + 4 scores of 4 bytes."""
    from random_rotation_kv_b200 import binding as B
    from random_rotation_kv_b200 import workloads as W
    stream = torch.cuda.current_stream(dev)
    rows = []
    for d in (64, 128, 256, 512):
        w = W.scores(d=d)
        t_len = w.x.shape[0]
        k = torch.from_numpy(w.flat()).to(dev)
        q = torch.from_numpy(w.extra["q"]).to(dev)
        for bits in (1, 2, 3, 4):
            codes, norms = B.rrq_encode(k, bits, 42)
            per_copy = codes.numel() + 4 * norms.numel() + 32 * t_len * 4
            copies = max(3, -(-(384 << 20) // per_copy))
            cs = [(codes, norms)] + [(codes.clone(), norms.clone()) for _ in range(copies - 1)]
            sc = [torch.empty(32, t_len, dtype=torch.float32, device=dev) for _ in range(copies)]
            ms = time_loop(torch, stream, lambda i: B.rrq_qk_scores(
                q, *cs[i % copies], 8, d, bits, 42, out=sc[i % copies]), reps)
            nkh = t_len * 8
            by = nkh * (d * bits // 8 + 4 + 16)
            rows.append({"d": d, "bits": bits, "us": 1e3 * ms, "gbs": by / ms / 1e6,
                         "frac_of_hbm": by / ms / 1e6 / peak, "copies": copies})
            del cs, sc, codes, norms
        del k
    return {"workload": "32 q heads x [131072 tokens x 8 kv heads], KV distribution, scale 1",
            "rows": rows}


def extra_kernels(torch, dev, flush, reps, peak, sel=None):
    """Other hot-path kernels on their own workloads (not part of the headline step),
    each timed as `reps` back-to-back launches whose inputs exceed L2 (the 1M-vector
    inputs are 268 MB; the scores rotate over 3 copies of its 71 MB cache)."""
    from random_rotation_kv_b200 import binding as B
    from random_rotation_kv_b200 import workloads as W
    stream = torch.cuda.current_stream(dev)
    mp = None
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            mp = json.load(f)
    except Exception:
        pass
    tc_peak = float(mp["bf16_tflops"]) if mp else 1590.0
    out = {}

    def want(name):
        return sel is None or name in sel

    w = W.scores()
    q = torch.from_numpy(w.extra["q"]).to(dev)
    nkh = w.x.shape[0] * 8

    # workload 5: scores of 32 query heads against 131072 tokens x 8 KV heads, 4-bit codes
    if want("qk_scores"):
        k = torch.from_numpy(w.flat()).to(dev)
        codes, norms = B.rrq_encode(k, 4, 42)
        del k
        cs = [codes] + [codes.clone() for _ in range(2)]
        ns = [norms] + [norms.clone() for _ in range(2)]
        scs = [torch.empty(32, w.x.shape[0], dtype=torch.float32, device=dev) for _ in range(3)]
        ms = time_loop(torch, stream,
                       lambda k: B.rrq_qk_scores(q, cs[k % 3], ns[k % 3], 8, 128, 4, 42, out=scs[k % 3]),
                       reps)
        by = nkh * (64 + 4) + 32 * w.x.shape[0] * 4
        out["qk_scores"] = {"workload": "32 q heads x [131072 tokens x 8 kv heads] d=128 b=4",
                            "us": 1e3 * ms, "bytes": by, "gbs": by / ms / 1e6,
                            "frac_of_hbm": by / ms / 1e6 / peak}
        del codes, norms, cs, ns, scs

        # one decode step of attention over a 4-bit K/V cache of the same shape
    if want("attention_decode"):
        kt = torch.from_numpy(w.flat()).to(dev)
        kc, kn_ = B.rrq_encode(kt, 4, 42)
        vc, vn_ = B.rrq_encode(kt, 4, 43)  # values: the same tensor under another rotation
        del kt
        caches = [(kc, kn_, vc, vn_), (kc.clone(), kn_.clone(), vc.clone(), vn_.clone())]  # 2 x 142 MB
        ao = torch.empty(32, 128, dtype=torch.float32, device=dev)
        ws = torch.zeros(B.rrq_attention_workspace_bytes(32, 8, 128, w.x.shape[0]), dtype=torch.uint8,
                         device=dev)
        ms = time_loop(torch, stream, lambda i: B.rrq_attention_decode(
            q, *caches[i % 2], 8, 128, 42, 43, scale=128 ** -0.5, out=ao, workspace=ws), reps)
        by = nkh * (64 + 4) * 2 + 32 * 128 * 4
        out["attention_decode"] = {"workload": "32 q heads over [131072 tokens x 8 kv heads] d=128, "
                                               "4-bit K and V codes",
                                   "us": 1e3 * ms, "bytes": by, "gbs": by / ms / 1e6,
                                   "frac_of_hbm": by / ms / 1e6 / peak}
        del caches, kc, kn_, vc, vn_

    # decode attention at the other shapes (the score kernel, then the fp32 value sums):
    # random codes and log-normal norms of 131072 tokens x 8 kv heads; the bytes count
    # the cache read once and the output, not the scores' round trip through the workspace
    if want("attention_shapes"):
        rows = w.x.shape[0] * 8
        g = torch.Generator(device=dev).manual_seed(77)
        lines = []
        for d, kb, vb in ((128, 2, 2), (128, 3, 3), (64, 4, 4), (256, 4, 4)):
            qd = torch.randn(32, d, device=dev, generator=g).half()
            caches = []
            for _ in range(2):
                caches.append((torch.randint(0, 256, (rows, d * kb // 8), device=dev, generator=g, dtype=torch.uint8),
                               torch.exp(torch.randn(rows, device=dev, generator=g) * 0.5) * 10,
                               torch.randint(0, 256, (rows, d * vb // 8), device=dev, generator=g, dtype=torch.uint8),
                               torch.exp(torch.randn(rows, device=dev, generator=g) * 0.5) * 10))
            ao = torch.empty(32, d, dtype=torch.float32, device=dev)
            ws = torch.zeros(B.rrq_attention_workspace_bytes(32, 8, d, w.x.shape[0], kb, vb), dtype=torch.uint8,
                             device=dev)
            ms = time_loop(torch, stream, lambda i: B.rrq_attention_decode(
                qd, *caches[i % 2], 8, d, 42, 43, k_bits=kb, v_bits=vb, scale=d ** -0.5, out=ao, workspace=ws),
                max(reps // 5, 5))
            by = rows * (d * kb // 8 + 4 + d * vb // 8 + 4) + 32 * d * 4
            lines.append({"d": d, "k_bits": kb, "v_bits": vb, "us": 1e3 * ms, "bytes": by,
                          "gbs": by / ms / 1e6, "frac_of_hbm": by / ms / 1e6 / peak})
            del caches, ws
        out["attention_shapes"] = {"workload": "32 q heads over [131072 tokens x 8 kv heads], random codes",
                                   "lines": lines}

        # unbiased scores on the same keys stored TurboQuant-style: 2-bit codes + QJL bits
    if want("qk_scores_qjl"):
        S = B.rrq_qjl_matrix(4242, 128, device=dev)
        k = torch.from_numpy(w.flat()).to(dev)
        sets = []
        for _ in range(3):  # 3 copies of 56 MB: larger than L2 in rotation
            c2, n2, b2, r2 = B.rrq_encode(k, 2, 42, qjl_S=S)
            sets.append((c2, n2, b2, r2))
        del k
        sc = [torch.empty(32, w.x.shape[0], dtype=torch.float32, device=dev) for _ in range(3)]
        ms = time_loop(torch, stream, lambda i: B.rrq_qk_scores_qjl(
            q, *sets[i % 3], S, 8, 128, 2, 42, out=sc[i % 3]), reps)
        by = nkh * (32 + 4 + 16 + 4) + 32 * w.x.shape[0] * 4
        out["qk_scores_qjl"] = {"workload": "32 q heads x [131072 tokens x 8 kv heads] d=128, "
                                            "2-bit codes + QJL bits (unbiased)",
                                "us": 1e3 * ms, "bytes": by, "gbs": by / ms / 1e6,
                                "frac_of_hbm": by / ms / 1e6 / peak}
        del sets, sc

    if want("qk_scores_sweep"):
        out["qk_scores_sweep"] = scores_sweep(torch, dev, reps, peak)

    if want("q4_0_rot") or want("ggml") or want("drive_1bit"):
        w = W.attnrot()
        x = torch.from_numpy(w.flat()).to(dev)
        n = x.shape[0]

    # workload 3: rotate-then-q4_0, 1,048,576 fp16 vectors
    if want("q4_0_rot"):
        blk = torch.empty(n, 72, dtype=torch.uint8, device=dev)
        xo = torch.empty_like(x)
        ms_e = time_loop(torch, stream, lambda k: B.rrq_q4_0_rot(x, 42, out=blk), reps)
        ms_d = time_loop(torch, stream, lambda k: B.rrq_q4_0_rot_decode(blk, 128, 42, out=xo), reps)
        by = n * (256 + 72)
        # reconstruction MSE over all 1,048,576 vectors, rotated and unrotated q4_0
        mse = {}
        for rot in (True, False):
            bq = B.rrq_q4_0_rot(x, 42, rotate=rot)
            xq = B.rrq_q4_0_rot_decode(bq, 128, 42, rotate=rot, out_dtype=torch.float32)
            mse[rot] = float(((xq.double() - x.double()) ** 2).mean())
            del bq, xq
        out["q4_0_rot"] = {"workload": "fp16 [131072 x 8 x 128], rotate + q4_0", "encode_us": 1e3 * ms_e,
                           "decode_us": 1e3 * ms_d, "encode_gbs": by / ms_e / 1e6,
                           "decode_gbs": by / ms_d / 1e6, "encode_frac_of_hbm": by / ms_e / 1e6 / peak,
                           "decode_frac_of_hbm": by / ms_d / 1e6 / peak,
                           "mse_rotated": mse[True], "mse_unrotated": mse[False],
                           "mse_rotated_over_unrotated": mse[True] / mse[False]}
        del blk, xo

    # the other GGML block types on the same vectors (rotate, then blocks of 32)
    if want("ggml"):
        for fmt in ("q4_1", "q5_0", "q5_1", "q8_0"):
            per = 4 * B.rrq_ggml_block_bytes(fmt)
            gb = torch.empty(n, per, dtype=torch.uint8, device=dev)
            xo = torch.empty_like(x)
            ms_e = time_loop(torch, stream, lambda k: B.rrq_ggml_rot(x, 42, fmt, out=gb), reps)
            ms_d = time_loop(torch, stream, lambda k: B.rrq_ggml_rot_decode(gb, 128, 42, fmt, out=xo), reps)
            by = n * (256 + per)
            out[f"{fmt}_rot"] = {"workload": f"fp16 [131072 x 8 x 128], rotate + {fmt}",
                                 "encode_us": 1e3 * ms_e, "decode_us": 1e3 * ms_d,
                                 "encode_gbs": by / ms_e / 1e6, "decode_gbs": by / ms_d / 1e6,
                                 "encode_frac_of_hbm": by / ms_e / 1e6 / peak,
                                 "decode_frac_of_hbm": by / ms_d / 1e6 / peak}
            del gb, xo

    # DRIVE one-bit encode (unbiased scale) of the same vectors, and the
    # one-bit decode back to fp16
    if want("drive_1bit"):
        dc = torch.empty(n, 16, dtype=torch.uint8, device=dev)
        ds = torch.empty(n, dtype=torch.float32, device=dev)
        xo = torch.empty_like(x)
        ms_e = time_loop(torch, stream,
                         lambda k: B.rrq_drive_encode(x, 42, True, codes=dc, scales=ds), reps)
        ms_d = time_loop(torch, stream, lambda k: B.rrq_decode(
            dc, ds, 128, 1, 42, codebook=[-1.0, 1.0], out=xo), reps)
        by = n * (256 + 16 + 4)
        out["drive_1bit"] = {"workload": "fp16 [131072 x 8 x 128], DRIVE sign + unbiased scale",
                             "encode_us": 1e3 * ms_e, "decode_us": 1e3 * ms_d,
                             "encode_gbs": by / ms_e / 1e6, "decode_gbs": by / ms_d / 1e6,
                             "encode_frac_of_hbm": by / ms_e / 1e6 / peak,
                             "decode_frac_of_hbm": by / ms_d / 1e6 / peak}
        del dc, ds, xo

    # workload 4: 2-bit codes + QJL sketch, 1,048,576 bf16 vectors (tcgen05 projection)
    if want("encode_qjl"):
        w = W.turbo()
        x = torch.from_numpy(w.flat()).to(dev).to(torch.bfloat16)
        n = x.shape[0]
        S = B.rrq_qjl_matrix(4242, 128, device=dev)
        cq = torch.empty(n, 32, dtype=torch.uint8, device=dev)
        nq = torch.empty(n, dtype=torch.float32, device=dev)
        qb = torch.empty(n, 16, dtype=torch.uint8, device=dev)
        rq = torch.empty(n, dtype=torch.float32, device=dev)
        ms = time_loop(torch, stream, lambda k: B.rrq_encode(
            x, 2, 42, codes=cq, norms=nq, qjl_S=S, qjl_bits=qb, qjl_rnorm=rq), reps)
        by = n * (256 + 32 + 4 + 16 + 4)
        flops = n * 2 * 2 * 128 * 128  # two fp16 MMA passes (residual split r_hi + r_lo)
        out["encode_qjl"] = {"workload": "bf16 [1048576 x 128], b=2 + QJL (2 fp16 MMA passes per tile)",
                             "us": 1e3 * ms, "gbs": by / ms / 1e6, "frac_of_hbm": by / ms / 1e6 / peak,
                             "tensor_tflops": flops / ms / 1e9,
                             "frac_of_tensor_peak": flops / ms / 1e9 / tc_peak}
    return out


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["rrq", "reference"], default="rrq")
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--ref-sample", type=int, default=16384,
                    help="largest number of vectors per reference (oracle) step")
    ap.add_argument("--ref-budget", type=float, default=90.0,
                    help="seconds of CPU the whole reference run should take")
    ap.add_argument("--settle-s", type=float, default=0.5,
                    help="seconds of untimed steps before timing, so clocks reach steady state")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip timing the other kernels (scores, q4_0, QJL) on their workloads")
    ap.add_argument("--extras", default="",
                    help="comma-separated subset of the other kernels and reports (qk_scores, "
                         "attention_decode, qk_scores_qjl, qk_scores_sweep, q4_0_rot, ggml, "
                         "drive_1bit, encode_qjl, reports); default all")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)  # at least 3 untimed warm-up steps, always
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
