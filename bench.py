"""Benchmark of the Hyena hot path on B200.

Workload: the order-2 Hyena operator at B=8, D=768, L=8192 with bf16 I/O and
fp32 FFT math (implicit filters 65->64->64->768).  One step is one pass of the
whole path over one batch: implicit filter generation (PE + MLP + decay),
filter spectra (zero-padded rFFT), and the fused FFT convolution with skip
term and gate -- three launches of this library's kernels.

Metric: achieved GB/s of compulsory HBM traffic per step (the operator's
inputs, output and filter spectra read once, plus the spectra written once by
the filter path), with ms per step and the fraction of the measured HBM peak.
Inputs stream 352 MB per step through a 126 MB L2, so no flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (independent batches, no collective on the data path: weak scaling); the
timed region is bracketed by barriers and the slowest rank's time counts.
``--impl reference`` times the float64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import hyena_workloads as hw  # noqa: E402

WORKLOAD = "c2"
L2_BYTES = 126 * 1024 * 1024


def workload_bytes(spec):
    """Compulsory bytes of one step and of one operator launch."""
    B, D, L = spec["B"], spec["D"], spec["L"]
    el = 2 if spec["dtype"] == "bf16" else 4
    K = spec["order"] - 1
    bins = 1
    while bins < L:
        bins *= 2
    bins = max(bins, 16) + 1
    sig = B * D * L * el
    spectra = K * D * bins * 8
    op = (1 + K) * sig + sig + spectra + K * D * 4          # v, x_k, y, H, Dskip
    step = op + spectra                                       # + spectra written by the filter path
    return step, op


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, t_begin=None, t_end=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.flush()
        rows = []
        with open(self.f.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                if t_begin is not None:
                    try:
                        import datetime
                        ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    except ValueError:
                        ts = None
                    if ts is not None and not (t_begin - 0.05 <= ts <= t_end + 0.05):
                        continue
                rows.append(parts)
        os.unlink(self.f.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import implicit_long_convolution_b200 as hy

    world, rank, local = dist_setup()
    w = hw.make(WORKLOAD, seed=hw.SEEDS[WORKLOAD] + 1000 * rank)
    s = w.spec
    B, D, L, K = s["B"], s["D"], s["L"], s["order"] - 1
    dev = torch.device("cuda", local)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    bf = lambda sig: torch.from_numpy(sig.bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    Ws, bs, alpha = [f32(a) for a in w.Ws], [f32(a) for a in w.bs], f32(w.alpha)
    Dsk = [f32(w.Dskip[k]) for k in range(K)]
    v, xs = bf(w.v), [bf(x) for x in w.xs]
    y = torch.empty_like(v)
    nb = hy.spectrum_bins(L)
    h = torch.empty((K * D, L), device=dev)
    H = torch.empty((K * D, nb), dtype=torch.complex64, device=dev)
    Hs = [H[k * D:(k + 1) * D] for k in range(K)]
    stream = torch.cuda.current_stream(dev)
    op_ev = []

    def step(record=False):
        hy.hyena_filter_gen(h, ndim=1, L=L, Ws=Ws, bs=bs, alpha=alpha, n_freq=s["F"], include_t=True)
        hy.hyena_filter_spectrum(h, H, rows=K * D, ndim=1, dims=[L])
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        hy.hyena_operator(v, xs, Hs, y, Dskips=Dsk)
        if record:
            e1.record(stream)
            op_ev.append((e0, e1))

    launches_per_step = 3
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.5)
    wall0 = time.time()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    ck = clocks.stop(wall0, wall1)
    ms = t0.elapsed_time(t1)
    op_ms = [a.elapsed_time(b) for a, b in op_ev]
    ms = max_over_ranks(ms, world)
    op_avg = max_over_ranks(sum(op_ms) / len(op_ms), world)

    step_bytes, op_bytes = workload_bytes(s)
    sec = ms / 1e3
    value = world * args.steps * step_bytes / sec / 1e9
    peak, peak_kind = measured_peaks()
    achieved = op_bytes / (op_avg / 1e3) / 1e9

    # end to end through the public API with host buffers: H2D of the step's
    # inputs from pinned memory, the path, D2H of the result
    hv = torch.from_numpy(w.v.bf16.view(np.int16)).view(torch.bfloat16).pin_memory()
    hx = [torch.from_numpy(x.bf16.view(np.int16)).view(torch.bfloat16).pin_memory() for x in w.xs]
    hy_out = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    e2e_steps = max(2, min(args.steps, 10))

    def e2e_step():
        v.copy_(hv, non_blocking=True)
        for xd, xh in zip(xs, hx):
            xd.copy_(xh, non_blocking=True)
        step()
        hy_out.copy_(y, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(a0.elapsed_time(a1) / e2e_steps, world)
    h2d = hv.numel() * 2 + sum(x.numel() * 2 for x in hx)
    d2h = hy_out.numel() * 2

    line = {
        "metric": "Hyena op GB/s (order-2, B8 D768 L8192, bf16 I/O, fp32 FFT math)",
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32 math, bf16 I/O",
        "data": "synthetic (seeded N(0,1) signals, random-init filter MLP)",
        "config": {"workload": "hyena order-2 operator B8 D768 L8192 bf16 (filters 65->64->64->768)",
                   "B": B, "D": D, "L": L, "order": K + 1,
                   "step": "filter_gen + filter_spectrum + hyena_operator",
                   "step_bytes": step_bytes, "operator_bytes": op_bytes,
                   "l2": "inputs larger than L2 (%.0f MB streamed per step vs 126 MB)" % (op_bytes / 1e6),
                   "parallelism": "replicas x%d" % world},
        "tokens_channels_per_s": round(world * args.steps * B * D * L / sec, 1),
        "operator_ms": round(op_avg, 4),
        "roofline": {"bound": "hbm", "kernel": "resident_conv_kernel<13,bf16>",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": None},
        "e2e": {"value": round(world * step_bytes / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": ck,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ oracle arm

def cpu_baseline(w, budget_s=12.0):
    """The float64 oracle as it stands on a bounded sample of the workload:
    the filter MLP for all L positions plus the direct O(L^2) gated chain on
    as many rows as fit the time budget.  Value in the metric's unit."""
    import oracle
    s = w.spec
    B, D, L, K = s["B"], s["D"], s["L"], s["order"] - 1
    step_bytes, _ = workload_bytes(s)
    rows_total = B * D
    t0 = time.perf_counter()
    h64 = oracle.filter_gen_1d(L, s["F"], True, w.Ws, w.bs, w.alpha)
    t_filter = time.perf_counter() - t0
    cores = oracle.threads()
    probe = max(cores, 8)
    t0 = time.perf_counter()
    oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], h64.reshape(K, D, L), w.Dskip,
                      rows=np.arange(probe))
    t_probe = time.perf_counter() - t0
    n = int(max(probe, min(rows_total, probe * max(1.0, (budget_s - t_filter) / max(t_probe, 1e-3)))))
    n = max(cores, (n // cores) * cores)
    rows = np.random.default_rng(0).choice(rows_total, n, replace=False)
    t0 = time.perf_counter()
    oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], h64.reshape(K, D, L), w.Dskip, rows=rows)
    t_rows = time.perf_counter() - t0
    # scale: the whole step = filter path once + all rows
    est_step = t_filter + t_rows * rows_total / n
    return {"value": round(step_bytes / est_step / 1e9, 6), "unit": "GB/s", "cores": cores,
            "kind": "oracle",
            "sample": "filter MLP on all %d positions + direct O(L^2) float64 chain on %d of %d rows "
                      "(%.1f s); value scales the sample to one whole step" % (L, n, rows_total,
                                                                               t_filter + t_rows)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = hw.make(WORKLOAD)
    budget = max(2.0, min(args.cpu_budget, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(w, budget_s=budget)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(w, budget_s=budget)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    step_bytes, _ = workload_bytes(w.spec)
    value = statistics.median(vals)
    line = {
        "impl": "reference",
        "metric": "Hyena op GB/s (order-2, B8 D768 L8192, bf16 I/O, fp32 FFT math)",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_bytes / (value * 1e9) * 1e3, 3) if value > 0 else None,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) signals, random-init filter MLP)",
        "config": {"workload": "hyena order-2 operator B8 D768 L8192 bf16 (filters 65->64->64->768)",
                   "B": 8, "D": 768, "L": 8192, "order": 2},
        "cpu_baseline": last,
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 1),
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
