"""Benchmark of the Hyena hot path on B200.

Default workload (the headline): the order-2 Hyena operator at B=8, D=768,
L=8192 with bf16 I/O and fp32 FFT math (implicit filters 65->64->64->768).
One step is one pass of the whole path over one batch: implicit filter
generation (PE + MLP + decay), filter spectra (zero-padded rFFT), and the
fused FFT convolution with skip term and gate -- all in this library's kernels.

Other workloads (``--workload``): c1 (order 2, B1 D16 L1024 fp32), c3 (order 3,
B1 D256 L=2^20 fp32, multi-pass), c4 (HyenaND 3-D, B2 D128 64^3 fp32,
FiLM filters), c5 (spectral gate, B4 H32 Dh64 L32768 bf16).

Metric: achieved GB/s of compulsory HBM traffic per step (inputs, outputs and
filter spectra read once, plus the spectra written once by the filter path),
with ms per step and, for the dominant kernel (the convolution), the fraction
of the measured HBM peak.  Every workload but c1 streams more than the 126 MB
L2 per step, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload c1|c2|c3|c4|c5]

Under torchrun (N > 1) every rank runs the same per-GPU workload on its own
GPU (independent batches, no collective on the data path: weak scaling); the
timed region is bracketed by barriers and the slowest rank's time counts.
``--impl reference`` times the float64 CPU oracle on a bounded sample.
"""
from __future__ import annotations

import argparse
import datetime
import json
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

DEFAULT_WORKLOAD = "c2"
DESCR = {
    "c1": "hyena order-2 operator B1 D16 L1024 fp32 (filters 17->32->16)",
    "c2": "hyena order-2 operator B8 D768 L8192 bf16 (filters 65->64->64->768)",
    "c3": "hyena order-3 operator B1 D256 L1048576 fp32 (filters 17->64->512)",
    "c4": "hyenaND order-2 3-D conv B2 D128 64^3 fp32 (FiLM from 8 register tokens; filters 24->64->128 on 128^3)",
    "c5": "spectral gate B4 H32 Dh64 L32768 bf16",
}


def spectrum_bins(L):
    m = 16
    while m < L:
        m *= 2
    return m + 1


def workload_bytes(spec):
    """(compulsory bytes of one step, of the convolution launch(es))."""
    sig = hw.signal_bytes(spec)
    if spec["kind"] == "operator":
        K, D = spec["order"] - 1, spec["D"]
        spectra = K * D * spectrum_bins(spec["L"]) * 8
        op = (1 + K) * sig + sig + spectra + K * D * 4
        return op + spectra, op
    if spec["kind"] == "nd":
        S = 2 * spec["grid"][0]
        spectra = spec["B"] * spec["D"] * S * S * (S // 2 + 1) * 8
        op = 2 * sig + sig + spectra
        return op + spectra, op
    gate = spec["H"] * (spec["L"] // 2 + 1) * 8
    op = 3 * sig + gate
    return op, op


# sources of the default (SIMT) on-chip convolution kernels; the opt-in
# tensor-core engine (resident_tc.cu, tcgen05.cuh) is not part of them
CONV_SOURCES = ["bulk_copy.cuh", "common.cuh", "fft_core.cuh", "resident.cuh", "resident_launch.cuh", "resident.cu",
                "resident_stream_bf16.cu", "resident_stream_f32.cu", "twiddle.cu", "twiddle.h"]


def conv_sources_digest():
    """sha256 over the sources of the on-chip convolution kernels."""
    import hashlib
    hsh = hashlib.sha256()
    for f in CONV_SOURCES:
        with open(os.path.join(ROOT, "implicit_long_convolution_b200", "csrc", f), "rb") as fh:
            hsh.update(fh.read())
    return hsh.hexdigest()


def recorded_traffic(kernel_key):
    """DRAM bytes per launch from the last ncu capture of this kernel, or None
    when the kernel's sources changed since (profiles/dram_traffic.json)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec or rec.get("sources_sha256") != conv_sources_digest():
        return None
    return rec.get("dram_bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region.

    Read-only NVML queries from a thread of this process every ~1 ms (so even
    a timed region of a few milliseconds has samples); nvidia-smi at 100 ms
    when NVML cannot be used.  Nothing is set on the GPU."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h): sw power cap, hw slowdown, sw / hw thermal
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40}

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.thread = None
        self.samples = []
        self.stop_flag = False
        self.f = None
        self.nvml = None
        self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.handle = self._handle(pynvml, index)
        except Exception:
            self.nvml = None

    @staticmethod
    def _handle(pynvml, index):
        """The NVML handle of CUDA device `index` (matched by UUID, so a
        CUDA_VISIBLE_DEVICES remap is honoured)."""
        try:
            import torch
            want = str(torch.cuda.get_device_properties(index).uuid).lower()
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = (u.decode() if isinstance(u, bytes) else u).lower()
                if u.replace("gpu-", "") == want.replace("gpu-", ""):
                    return h
        except Exception:
            pass
        return pynvml.nvmlDeviceGetHandleByIndex(index)

    def _poll(self):
        nv, h = self.nvml, self.handle
        reasons_fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self.stop_flag:
            try:
                self.samples.append((time.time(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     int(reasons_fn(h))))
            except Exception:
                pass
            time.sleep(0.001)

    def start(self):
        if self.nvml is not None:
            import threading
            try:
                self.max_mhz = self.nvml.nvmlDeviceGetMaxClockInfo(self.handle, self.nvml.NVML_CLOCK_SM)
            except Exception:
                self.max_mhz = None
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
            return
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, t_begin=None, t_end=None):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(5)
            rows = [r for r in self.samples
                    if t_begin is None or (t_begin - 0.002 <= r[0] <= t_end + 0.002)]
            if not rows:
                return None
            reasons = sorted({n for r in rows for n, b in self.BITS.items() if r[2] & b})
            return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(rows), "source": "nvml in-process, ~1 ms"}
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
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "source": "nvidia-smi, 100 ms"}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The slowest rank's value (used for every timed quantity)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(name, rank):
    """Each rank draws its own batch of the same per-GPU workload."""
    return hw.SEEDS[name] + 1000 * rank


def job_value(world, steps, step_bytes, max_ms):
    """Whole-job GB/s: the bytes of every rank's steps over the slowest rank's time."""
    return world * steps * step_bytes / (max_ms / 1e3) / 1e9


def workload_config(name, s, world, over=None):
    """The `config` object of a bench line (the same for both arms)."""
    step_bytes, op_bytes = workload_bytes(s)
    cfg = {"workload": DESCR[name] + (" [D=%d profiling case]" % s["D"] if over else "")}
    cfg.update({k: v for k, v in s.items() if k in ("B", "D", "L", "order", "H", "Dh", "grid")})
    cfg["io_dtype"] = s["dtype"]
    cfg.update({"step": ("spectral_gate" if s["kind"] == "gate" else
                         "register_film + filter_gen + filter_spectrum + convolution" if s.get("registers")
                         else "filter_gen + filter_spectrum + convolution"),
                "step_bytes": step_bytes, "conv_bytes": op_bytes,
                "l2": ("inputs larger than L2 (%.0f MB streamed per step vs 126 MB); no flush" % (op_bytes / 1e6)
                       if op_bytes > 126e6 else "inputs smaller than L2 (no flush): launch-bound case"),
                "parallelism": "independent replicas x%d (no data-path collective)" % world})
    return cfg


# ------------------------------------------------------------------ setups

class Setup:
    """Device state of one workload: spectra() runs the filter rows of the
    path, op() the convolution; inputs (device, host signal) feed the
    end-to-end run."""

    def __init__(self):
        self.inputs = []
        self.output = None
        self.launches = 0
        self.kernel = ""
        self.host_op = None      # op() on host buffers through the host-buffer entry point


def setup_operator(w, dev, hy, torch):
    s = w.spec
    B, D, L, K = s["B"], s["D"], s["L"], s["order"] - 1
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    if s["dtype"] == "bf16":
        sig = lambda x: torch.from_numpy(x.bf16.view(np.int16)).view(torch.bfloat16).to(dev)
        code = hy.HY_BF16
    else:
        sig = lambda x: torch.from_numpy(np.ascontiguousarray(x.f32)).to(dev)
        code = hy.HY_F32
    Ws, bs, alpha = [f32(a) for a in w.Ws], [f32(a) for a in w.bs], f32(w.alpha)
    Dsk = [f32(w.Dskip[k]) for k in range(K)]
    v, xs = sig(w.v), [sig(x) for x in w.xs]
    y = torch.empty_like(v)
    nb = hy.spectrum_bins(L)
    h = torch.empty((K * D, L), device=dev)
    H = torch.empty((K * D, nb), dtype=torch.complex64, device=dev)
    Hs = [H[k * D:(k + 1) * D] for k in range(K)]
    wsf = hy.filter_spectrum_workspace(K * D, 1, [L])
    wso = hy.operator_workspace(K + 1, B, D, L, code)
    ws = torch.empty(max(wsf, wso, 1), dtype=torch.uint8, device=dev)
    st = Setup()

    def spectra():
        hy.hyena_filter_gen(h, ndim=1, L=L, Ws=Ws, bs=bs, alpha=alpha, n_freq=s["F"], include_t=True)
        hy.hyena_filter_spectrum(h, H, rows=K * D, ndim=1, dims=[L], ws=ws if wsf else None)

    def op():
        hy.hyena_operator(v, xs, Hs, y, Dskips=Dsk, ws=ws if wso else None)

    wsh = torch.empty(hy.operator_host_workspace(K + 1, B, D, L, code), dtype=torch.uint8, device=dev)

    def host_op(hosts, out_h):
        hy.hyena_operator_host(hosts[0], hosts[1:], Hs, out_h, Dskips=Dsk, ws=wsh)

    st.spectra, st.op, st.host_op = spectra, op, host_op
    st.inputs = [(v, w.v)] + list(zip(xs, w.xs))
    st.output = y
    M = nb - 1
    # multi-pass chunks: ~104 MB of 8-byte points per chunk (the workspace
    # holds two chunk buffers when there is more than one chunk)
    def chunk_rows(rows):
        return max(1, min(rows, (104 << 20) // (8 * M)))
    if wso:
        op_l = -(-(B * D) // chunk_rows(B * D)) * (1 + 2 * K)
        st.kernel = "multi-pass colpass/rowpass kernels (M=2^%d)" % (M.bit_length() - 1)
    else:
        op_l = 1
        # one order over power-of-two rows runs a persistent streaming kernel;
        # bf16 rows of 8192 take the one with tensor-core radix-32 stages
        stream = K == 1 and L == M and M >= 64
        tensor = stream and L == 8192 and s["dtype"] == "bf16" and os.environ.get("HYENA_FFT_ENGINE") == "tensor"
        st.kernel = "%s<M=2^%d>" % ("resident_tc_kernel" if tensor else
                                    "resident_stream_kernel" if stream else "resident_conv_kernel",
                                    M.bit_length() - 1)
    spec_l = 2 * -(-(K * D) // chunk_rows(K * D)) if wsf else 1
    st.launches = 1 + spec_l + op_l
    return st


def setup_nd(w, dev, hy, torch):
    s = w.spec
    B, D, g = s["B"], s["D"], s["grid"][0]
    S = 2 * g
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    Ws, bs, alpha = [f32(a) for a in w.Ws], [f32(a) for a in w.bs], f32(w.alpha)
    if w.reg is not None:
        # input conditioning: z(x) from the register activations drives FiLM
        H1 = s["hidden"][0]
        gm = torch.empty((B, H1), device=dev)
        bt = torch.empty((B, H1), device=dev)
        reg, rq, fW, fb = f32(w.reg), f32(w.reg_query), f32(w.film_W), f32(w.film_b)
        condition = lambda: hy.hyena_register_film(reg, fW, gm, bt, query=rq, b_film=fb)
    else:
        gm, bt = f32(w.film_gamma), f32(w.film_beta)
        condition = lambda: None
    u, x1 = f32(w.v.f32), f32(w.xs[0].f32)
    y = torch.empty_like(u)
    h = torch.empty((B, D, S, S, S), device=dev)
    H = torch.empty((B, D, S, S, S // 2 + 1), dtype=torch.complex64, device=dev)
    wsf = hy.filter_spectrum_workspace(B * D, 3, [g, g, g])
    wsc = hy.nd_conv_workspace([g, g, g], B, D)
    ws = torch.empty(max(wsf, wsc, 1), dtype=torch.uint8, device=dev)
    st = Setup()

    def spectra():
        condition()
        hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=Ws, bs=bs, alpha=alpha, n_freq=s["F"],
                            film_gamma=gm, film_beta=bt, n_sets=B)
        hy.hyena_filter_spectrum(h, H, rows=B * D, ndim=3, dims=[g, g, g], ws=ws)

    def op():
        hy.hyena_nd_conv(u, H, y, H_batch_stride=D * S * S * (S // 2 + 1), gate=x1, ws=ws)

    wsh = torch.empty(hy.nd_conv_host_workspace([g, g, g], B, D), dtype=torch.uint8, device=dev)

    def host_op(hosts, out_h):
        hy.hyena_nd_conv_host(hosts[0], H, out_h, H_batch_stride=D * S * S * (S // 2 + 1), gate=hosts[1], ws=wsh)

    st.spectra, st.op, st.host_op = spectra, op, host_op
    st.inputs = [(u, w.v), (x1, w.xs[0])]
    st.output = y
    per_c = g * S * (S // 2 + 1) * 8
    per_s = S * S * (S // 2 + 1) * 8
    # 3-D chunks: ~80 MB of transform planes (the workspace holds two chunk
    # buffers when there is more than one chunk)
    def chunks(per):
        return -(-(B * D) // max(1, min(B * D, (80 << 20) // per)))
    st.launches = (2 if w.reg is not None else 1) + 2 * chunks(per_s) + 3 * chunks(per_c)
    st.kernel = "nd_fwd_plane/nd_xpass/nd_inv_plane<S=%d>" % S
    return st


def setup_gate(w, dev, hy, torch):
    s = w.spec
    sig = lambda x: torch.from_numpy(x.bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    x, x2 = sig(w.v), sig(w.xs[0])
    g = torch.from_numpy(w.gate).to(dev)
    y = torch.empty_like(x)
    st = Setup()
    st.spectra = lambda: None

    def op():
        hy.spectral_gate(x, g, y, x2=x2)

    wsh = torch.empty(hy.spectral_gate_host_workspace(s["B"], s["H"], s["Dh"], s["L"], hy.HY_BF16),
                      dtype=torch.uint8, device=dev)

    def host_op(hosts, out_h):
        hy.spectral_gate_host(hosts[0], g, out_h, x2=hosts[1], ws=wsh)

    st.op, st.host_op = op, host_op
    st.inputs = [(x, w.v), (x2, w.xs[0])]
    st.output = y
    st.launches = 1
    st.kernel = "resident_stream_kernel<M=2^%d, circular>" % ((s["L"] // 2).bit_length() - 1)
    return st


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import implicit_long_convolution_b200 as hy

    world, rank, local = dist_setup()
    name = args.workload
    over = {"D": args.channels} if args.channels else {}
    w = hw.make(name, seed=rank_seed(name, rank), **over)
    s = w.spec
    dev = torch.device("cuda", local)
    setup = {"operator": setup_operator, "nd": setup_nd, "gate": setup_gate}[s["kind"]]
    st = setup(w, dev, hy, torch)
    stream = torch.cuda.current_stream(dev)
    op_ev = []

    def step(record=False):
        st.spectra()
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        st.op()
        if record:
            e1.record(stream)
            op_ev.append((e0, e1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = args.steps
    if steps <= 0:   # size the timed region to about one second
        ta, tb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ta.record(stream)
        step()
        tb.record(stream)
        torch.cuda.synchronize()
        steps = int(max(10, min(5000, 1000.0 / max(ta.elapsed_time(tb), 1e-3))))
        steps = int(max_over_ranks(steps, world))
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.5)
    wall0 = time.time()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        step(record=True)
    t1.record(stream)
    torch.cuda.synchronize()
    wall1 = time.time()
    barrier(world)
    ck = clocks.stop(wall0, wall1)
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    op_ms = [a.elapsed_time(b) for a, b in op_ev]
    op_avg = max_over_ranks(sum(op_ms) / len(op_ms), world)

    step_bytes, op_bytes = workload_bytes(s)
    sec = ms / 1e3
    value = job_value(world, steps, step_bytes, ms)
    peak, peak_kind = measured_peaks()
    achieved = op_bytes / (op_avg / 1e3) / 1e9

    # end to end through the public API with host buffers: H2D of the step's
    # input signals from pinned memory, the whole step, D2H of the result
    hosts = []
    for dvc, sg in st.inputs:
        if dvc.dtype == torch.bfloat16:
            t = torch.from_numpy(np.ascontiguousarray(sg.bf16.view(np.int16))).view(torch.bfloat16)
        else:
            t = torch.from_numpy(np.ascontiguousarray(sg.f32))
        hosts.append(t.pin_memory())
    out_h = torch.empty(st.output.shape, dtype=st.output.dtype).pin_memory()
    e2e_steps = max(2, min(steps, 10))

    def e2e_step():
        if st.host_op is not None:
            # filters and spectra on the device, then the path over host
            # buffers: copies in, compute and copies out overlap chunk by chunk
            st.spectra()
            st.host_op(hosts, out_h)
            return
        for (dvc, _), hst in zip(st.inputs, hosts):
            dvc.copy_(hst, non_blocking=True)
        step()
        out_h.copy_(st.output, non_blocking=True)

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
    h2d = sum(hh.numel() * hh.element_size() for hh in hosts)
    d2h = out_h.numel() * out_h.element_size()

    cfg = workload_config(name, s, world, over)
    el = 2 if s["dtype"] == "bf16" else 4
    line = {
        "metric": "Hyena op GB/s (%s)" % cfg["workload"],
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms / steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic (seeded N(0,1) signals, random-init filter MLP)",
        "config": cfg,
        "tokens_channels_per_s": round(world * steps * (hw.signal_bytes(s) // el) / sec, 1),
        "conv_ms": round(op_avg, 4),
        "roofline": {"bound": "hbm", "kernel": st.kernel,
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": recorded_traffic(name) if "resident_stream" in st.kernel else None},
        "e2e": {"value": round(world * step_bytes / (e2e_ms / 1e3) / 1e9, 2), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": st.launches * steps,
        "clocks": ck,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ oracle arm

class CpuSample:
    """One bounded sample of a workload, run by the float64 oracle (the
    direct definitions) and by the naive float64 FFT reference.

    `run_oracle()` / `run_fft()` each execute the sample once; `frac` is the
    sample's share of the step's elements, so `frac * step_bytes` are the
    compulsory bytes of the elements the sample produces and a rate is those
    bytes over the measured time.  Nothing is extrapolated."""

    def __init__(self, w):
        import oracle
        self.w = w
        s = w.spec
        kind = s["kind"]
        self.step_bytes = workload_bytes(s)[0]
        if kind == "operator":
            B, D, L, K = s["B"], s["D"], s["L"], s["order"] - 1
            rows_total = B * D
            if L <= 16384:
                # whole rows: the direct O(L^2) chain and the FFT route on the same rows
                # (about one second of the direct chain on 16 cores at L = 8192)
                n_rows = min(rows_total, max(16, (768 * 8192 ** 2) // (L * L)))
                rows = np.random.default_rng(0).permutation(rows_total)[:n_rows]
                self.frac = rows.size / rows_total
                self.fft_frac = self.frac
                self.desc = ("filter MLP on all %d positions + the direct O(L^2) float64 chain on %d of %d "
                             "whole rows" % (L, rows.size, rows_total))
                self.fft_desc = ("filter MLP on all %d positions + the naive radix-2 FFT chain (n = %d, "
                                 "filter transform per row) on the same %d rows" % (L, 2 * (spectrum_bins(L) - 1),
                                                                                     rows.size))
                fft_rows = rows
                T = L
            else:
                # long rows: the direct chain on a prefix (causal: a prefix needs input prefixes only);
                # the FFT route needs whole rows
                T = min(L, 32768)
                rows = np.arange(min(rows_total, max(oracle.threads(), 16)))
                fft_rows = np.arange(min(rows_total, 2))
                self.frac = rows.size * T / (rows_total * L)
                self.fft_frac = fft_rows.size / rows_total
                self.desc = ("filter MLP on all %d positions + the direct O(T^2) float64 chain on the first "
                             "T = %d samples of %d of %d rows (a longer prefix costs more per sample)"
                             % (L, T, rows.size, rows_total))
                self.fft_desc = ("filter MLP on all %d positions + the naive radix-2 FFT chain (n = %d) on %d of "
                                 "%d whole rows" % (L, 2 * (spectrum_bins(L) - 1), fft_rows.size, rows_total))
            v = w.v.f32
            xs = [x.f32 for x in w.xs]

            def filt():
                return oracle.filter_gen_1d(L, s["F"], True, w.Ws, w.bs, w.alpha).reshape(K, D, L)

            self.run_oracle = lambda: oracle.hyena_rows(v, xs, filt(), w.Dskip, rows=rows, T=T)
            self.run_fft = lambda: oracle.fftref_hyena_rows(v, xs, filt(), w.Dskip, rows=fft_rows)
        elif kind == "nd":
            B, D, g = s["B"], s["D"], s["grid"][0]
            S = 2 * g
            nvox = g ** 3
            pts = np.random.default_rng(0).permutation(nvox)[:min(nvox, 2048)]
            b, d = 0, 0
            self.frac = pts.size / (B * D * nvox)
            self.fft_frac = 1 / (B * D)
            self.desc = ("one slab's kernel from the filter MLP on the whole %d^3 transform grid (all %d channels "
                         "of sample 0) + the direct N-D sum at %d of its %d voxels" % (S, D, pts.size, nvox))
            self.fft_desc = ("the same kernel + the naive 3-D FFT route (1-D radix-2 FFTs along each axis of the "
                             "%d^3 grid) on that whole slab" % S)

            def kern():
                if w.reg is not None:      # z(x) from the registers, then FiLM
                    gm, bt, _, _ = oracle.register_film(w.reg[b:b + 1], w.reg_query, None, w.film_W, w.film_b)
                else:
                    gm, bt = w.film_gamma[b:b + 1], w.film_beta[b:b + 1]
                return oracle.filter_gen_3d(g, False, s["F"], w.Ws, w.bs, gm, bt, w.alpha)

            vs, x1 = w.v.f32[b, d], w.xs[0].f32[b, d]
            self.run_oracle = lambda: oracle.nd_conv_points(kern()[d], vs, x1, 0.0, pts, False)
            self.run_fft = lambda: oracle.fftref_nd_conv(kern()[d:d + 1], [0], vs[None], x1[None], False)
        else:
            B, H, Dh, L = s["B"], s["H"], s["Dh"], s["L"]
            rows_total = B * H * Dh
            head = 0
            n_rows = max(oracle.threads(), 16)
            x1 = w.v.f32.reshape(rows_total, L)
            x2 = w.xs[0].f32.reshape(rows_total, L)
            rows = np.arange(n_rows)                        # sample 0, head 0: channels 0..n_rows-1
            fft_rows = np.arange(min(Dh * 4, rows_total))   # sample 0, heads 0..3
            self.frac = rows.size / rows_total
            self.fft_frac = fft_rows.size / rows_total
            self.desc = ("the gate's circular kernel of one head by the direct inverse DFT + the direct O(L^2) "
                         "circular convolution on %d of %d rows" % (rows.size, rows_total))
            self.fft_desc = "the naive radix-2 FFT route on %d of %d rows" % (fft_rows.size, rows_total)

            def oracle_run():
                kap = oracle.gate_kernel(w.gate[head])
                return oracle.circular_conv_rows(kap[None], np.zeros(rows.size, np.int64), x1[rows], x2[rows])

            self.run_oracle = oracle_run
            gidx = (fft_rows // Dh) % H
            self.run_fft = lambda: oracle.fftref_gate_rows(w.gate, gidx, x1[fft_rows], x2[fft_rows])

    def time(self, which):
        fn = self.run_oracle if which == "oracle" else self.run_fft
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    def rate(self, which, seconds):
        frac = self.frac if which == "oracle" else self.fft_frac
        return self.step_bytes * frac / seconds / 1e9


def cpu_baseline(w):
    """The float64 oracle as it stands, and the naive float64 FFT reference,
    each timed once on a bounded sample of the workload on this host's
    cores.  value = compulsory bytes of the sample's elements / time."""
    import oracle
    cs = CpuSample(w)
    cores = oracle.threads()
    t_o = cs.time("oracle")
    t_f = cs.time("fft")
    return {"value": round(cs.rate("oracle", t_o), 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "%s (%.2f s); value = the compulsory bytes of the sampled elements / time" % (cs.desc, t_o),
            "fft_reference": {"value": round(cs.rate("fft", t_f), 6), "unit": "GB/s", "cores": cores,
                              "kind": "naive float64 FFT reference",
                              "sample": "%s (%.2f s)" % (cs.fft_desc, t_f)}}


def run_reference(args):
    """The reference arm: the float64 oracle as it stands, on this host's
    cores.  Every step runs the same bounded sample of the workload (see
    CpuSample); ms_per_step is the measured time of one such step and value
    the sample's compulsory bytes over it.  Under torchrun only rank 0 runs."""
    import oracle
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.workload
    w = hw.make(name)
    cs = CpuSample(w)
    for _ in range(args.warmup):
        cs.time("oracle")
    t0 = time.perf_counter()
    times = [cs.time("oracle") for _ in range(args.steps)]
    wall = time.perf_counter() - t0
    t_f = cs.time("fft")
    per_step = sum(times) / len(times)
    value = cs.rate("oracle", per_step)
    s = w.spec
    cores = oracle.threads()
    line = {
        "impl": "reference",
        "metric": "Hyena op GB/s (%s)" % DESCR[name],
        "value": round(value, 6), "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_step * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) signals, random-init filter MLP)",
        "config": workload_config(name, s, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: %s; value = the compulsory bytes of the sampled elements "
                                   "(%.4f of the step) / the measured step time" % (cs.desc, cs.frac),
                         "fft_reference": {"value": round(cs.rate("fft", t_f), 6), "unit": "GB/s",
                                           "cores": cores, "kind": "naive float64 FFT reference",
                                           "sample": "%s (%.2f s, once)" % (cs.fft_desc, t_f)}},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": round(wall, 4),
    }
    print(json.dumps(line), flush=True)


def run_projection(args):
    """The input projection at the operator workload's width (B8 L8192,
    768 -> 2 x 768 channels, bf16): one launch of the library's tcgen05 GEMM
    with the bias fused into its epilogue, timed with CUDA events; TFLOP/s
    against the measured bf16 GEMM peak (burst)."""
    import torch
    import implicit_long_convolution_b200 as hy
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    B, L, C, D, n_out = 8, 8192, 768, 768, 2
    g = torch.Generator(device=dev)
    g.manual_seed(rank_seed("c2", rank))
    x = torch.randn((B, L, C), device=dev, generator=g).to(torch.bfloat16)
    W = (torch.randn((n_out * D, C), device=dev, generator=g) / C ** 0.5).to(torch.bfloat16)
    bias = torch.randn(n_out * D, device=dev, generator=g) * 0.1
    outs = [torch.empty((B, D, L), dtype=torch.bfloat16, device=dev) for _ in range(n_out)]
    ws = torch.empty(hy.projection_workspace(), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    run = lambda: hy.hyena_projection(x, W, outs, bias=bias, ws=ws)
    for _ in range(max(3, args.warmup)):
        run()
    steps = args.steps if args.steps > 0 else 200
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        run()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    flops = 2.0 * B * L * C * n_out * D
    tf = world * flops / (ms / 1e3) / 1e12
    peak, peak_kind = 1590.0, "fallback"
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            peak, peak_kind = float(json.load(f)["bf16_tflops"]), "measured"
    if rank == 0:
        print(json.dumps({
            "metric": "input projection TFLOP/s (B8 L8192, 768 -> 2 x 768, bf16, channel-major outputs + bias)",
            "value": round(tf, 1), "unit": "TFLOP/s", "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "roofline": {"bound": "tensor", "kernel": "proj_tc_kernel", "achieved": round(tf / world, 1),
                         "peak": peak, "unit": "TFLOP/s", "frac": round(tf / world / peak, 4),
                         "peak_kind": peak_kind, "traffic": None},
            "config": {"workload": "hyena input projection at the order-2 operator width",
                       "B": B, "L": L, "C": C, "D": D, "n_out": n_out,
                       "accumulate": "f32"}}), flush=True)


def run_backward(args):
    """The operator's backward pass on the order-2 operator workload (B8 D768
    L8192, bf16 signals): dv, dx_1, dh_1 and dD_1 from dy, with the forward
    recomputed inside.  GB/s = compulsory bytes (v, x_1, dy and the spectra
    read; dv, dx_1 and dh_1 written) / time."""
    import torch
    import implicit_long_convolution_b200 as hy
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    w = hw.make("c2", seed=rank_seed("c2", rank), with_signals=True)
    s = w.spec
    B, D, L = s["B"], s["D"], s["L"]
    bf = lambda sig: torch.from_numpy(sig.bf16.view(np.int16)).view(torch.bfloat16).to(dev)
    v, x1 = bf(w.v), bf(w.xs[0])
    dy = torch.randn((B, D, L), device=dev).to(torch.bfloat16)
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(dev)
    Ws, bs, alpha = [f32(a) for a in w.Ws], [f32(a) for a in w.bs], f32(w.alpha)
    h = torch.empty((D, L), device=dev)
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=Ws, bs=bs, alpha=alpha, n_freq=s["F"], include_t=True)
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device=dev)
    hy.hyena_filter_spectrum(h, H, rows=D, ndim=1, dims=[L])
    dsk = [f32(w.Dskip[0])]
    dv, dx = torch.empty_like(v), [torch.empty_like(v)]
    dh, dD = [torch.empty((D, L), device=dev)], [torch.empty(D, device=dev)]
    ws = torch.empty(hy.operator_backward_workspace(2, B, D, L, hy.HY_BF16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    run = lambda: hy.hyena_operator_backward(v, [x1], [H], dy, dv, dx, Dskips=dsk, dhs=dh, dDs=dD, ws=ws)
    for _ in range(max(3, args.warmup)):
        run()
    steps = args.steps if args.steps > 0 else 50
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        run()
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    nb = hy.spectrum_bins(L)
    sig_bytes = B * D * L * 2
    step_bytes = 5 * sig_bytes + D * nb * 8 + D * L * 4 + D * 4
    if rank == 0:
        print(json.dumps({
            "metric": "Hyena op backward GB/s (order-2 operator B8 D768 L8192 bf16: dv, dx1, dh1, dD1)",
            "value": round(world * step_bytes / (ms / 1e3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "hyena order-2 operator backward B8 D768 L8192 bf16", "B": B, "D": D, "L": L,
                       "io_dtype": "bf16", "step_bytes": step_bytes}}), flush=True)


def run_decode(args):
    """One streaming decode step of the spectral gate at the gate workload's
    shape (B4 H32 Dh64, n = 32768, bf16 tokens): the prefix-FFT cache of all
    8192 rows is read and written once per step.  GB/s = (cache read + write,
    gate, the step's x, x2 and y) / time."""
    import torch
    import implicit_long_convolution_b200 as hy
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    B, Hh, Dh, n = 4, 32, 64, 32768
    nb = n // 2 + 1
    g = torch.randn((Hh, nb), dtype=torch.complex64, device=dev)
    cache = torch.zeros((B, Hh, Dh, nb), dtype=torch.complex64, device=dev)
    x = torch.randn((B, Hh, Dh), device=dev).to(torch.bfloat16)
    x2 = torch.randn_like(x)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)
    for p in range(max(3, args.warmup)):
        hy.spectral_gate_decode(x, g, cache, y, pos=p, x2=x2)
    steps = args.steps if args.steps > 0 else 100
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        hy.spectral_gate_decode(x, g, cache, y, pos=(args.warmup + i) % n, x2=x2)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1), world) / steps
    rows = B * Hh * Dh
    step_bytes = 2 * rows * nb * 8 + Hh * nb * 8 + 3 * rows * 2
    if rank == 0:
        print(json.dumps({
            "metric": "spectral gate streaming decode GB/s (prefix-FFT cache, B4 H32 Dh64 n32768, bf16 tokens)",
            "value": round(world * step_bytes / (ms / 1e3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "tokens_per_s": round(world * B / (ms / 1e3), 1),
            "config": {"workload": "spectral gate decode step B4 H32 Dh64 n32768", "B": B, "H": Hh, "Dh": Dh,
                       "n": n, "io_dtype": "bf16", "step_bytes": step_bytes}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=0, help="timed steps (0: size the region to ~1 s)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(DESCR), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--decode", action="store_true",
                    help="time one streaming decode step of the spectral gate (prefix-FFT cache) instead")
    ap.add_argument("--backward", action="store_true",
                    help="time the operator's backward pass on the order-2 operator workload instead")
    ap.add_argument("--projection", action="store_true",
                    help="time the input projection at the operator workload's width instead")
    ap.add_argument("--channels", type=int, default=0,
                    help="override the channel count D (smaller cases for profiler captures)")
    args = ap.parse_args()
    if args.channels and hw.WORKLOADS[args.workload]["kind"] == "gate":
        ap.error("--channels applies to the operator and N-D workloads")
    if args.impl == "reference":
        if args.steps <= 0:
            args.steps = 3
        run_reference(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.projection:
        run_projection(args)
        return
    if args.backward:
        run_backward(args)
        return
    if args.decode:
        run_decode(args)
        return
    run_ours(args)


if __name__ == "__main__":
    main()
