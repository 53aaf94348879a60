"""Seeded synthetic inputs for the Hyena hot path.

Shared by the tests, the benchmark and the smoke check, and by both sides of
every parity comparison (the CUDA library and the float64 oracle).  This
module holds random draws, their packing and the workload shapes only -- none
of the method's arithmetic -- and imports neither the product package nor the
oracle.

Recipe (numpy PCG64, ``default_rng(seed)``; seed = workload index 1..5 unless
overridden), drawn in this fixed order:

1. filter-MLP weights and biases, layer by layer: W_l, b_l ~ U(-1/sqrt(fan_in),
   +1/sqrt(fan_in)), float32;
2. decay rates alpha ~ U[lo, hi] per output column (order x channel), float32;
3. skip weights D ~ N(0, 1) per (order, channel), float32 (workloads with a
   skip term only);
4. FiLM parameters gamma_b, beta_b ~ N(0, 0.1^2) per sample on the first
   hidden layer (N-D workload), or the spectral gate a ~ N(0,1), phi ~
   U[-pi, pi] per (head, bin), packed as g = sigmoid(a) * exp(i phi) and
   rounded to complex64 (gate workload);
5. the signals: v then x_1, x_2, ... (or x1 then x2 for the gate), N(0, 1)
   float32, rounded to bfloat16 (round-to-nearest-even) for bf16 workloads --
   the rounded values are the inputs both sides see;
6. (N-D workload with ``registers=R``) register activations (B, R, C) ~ N(0,1),
   the pooling query ~ N(0, 1/C), the FiLM map W ~ U(+-0.1/sqrt(C)) of shape
   (2 hidden0, C) and its bias ~ N(0, 0.01^2): the input conditioning that
   replaces the drawn gamma/beta of step 4 when a test or the benchmark asks
   for it.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# The five workloads.  Shapes, widths and ranges follow the workload
# definitions; "F" is the number of sinusoid frequencies (2F features).
WORKLOADS = {
    # order-2 operator, fp32, small: B1 D16 L1024, PE 1+2*8=17, MLP 17->32->16
    "c1": dict(kind="operator", order=2, dtype="f32", B=1, D=16, L=1024, F=8, include_t=True,
               hidden=[32], alpha=(0.5, 3.0), skip=True),
    # order-2 operator at the ~153M-model width: B8 D768 L8192 bf16, MLP 65->64->64->768
    "c2": dict(kind="operator", order=2, dtype="bf16", B=8, D=768, L=8192, F=32, include_t=True,
               hidden=[64, 64], alpha=(0.3, 5.0), skip=True),
    # order-3 operator at 1M length: B1 D256 L2^20 fp32, MLP 17->64->(2*256)
    "c3": dict(kind="operator", order=3, dtype="f32", B=1, D=256, L=1 << 20, F=8, include_t=True,
               hidden=[64], alpha=(0.1, 2.0), skip=True),
    # order-2 gated 3-D global convolution: B2 D128 64^3 fp32, per-sample FiLM filters
    # (conditioned on the input through 8 register tokens of width 64)
    "c4": dict(kind="nd", order=2, dtype="f32", B=2, D=128, grid=(64, 64, 64), F=4,
               hidden=[64], alpha=(0.5, 3.0), skip=False, film=True, circular=False,
               registers=8, register_width=64),
    # spectral-gating token mixer: B4 H32 Dh64 L32768 bf16
    "c5": dict(kind="gate", dtype="bf16", B=4, H=32, Dh=64, L=32768),
}

SEEDS = {"c1": 1, "c2": 2, "c3": 3, "c4": 4, "c5": 5}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits (uint16) to float32 exactly."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class Signal:
    """One input tensor: float32 values (exactly the values both sides use)
    and, for bf16 workloads, the bfloat16 bit pattern the device receives."""
    f32: np.ndarray
    bf16: Optional[np.ndarray] = None

    def device_array(self, dtype: str) -> np.ndarray:
        return self.bf16 if dtype == "bf16" else self.f32


@dataclasses.dataclass
class Workload:
    name: str
    spec: dict
    Ws: list            # filter MLP weights, float32 (out x in)
    bs: list            # biases, float32
    alpha: Optional[np.ndarray] = None   # (n_out,) float32
    Dskip: Optional[np.ndarray] = None   # (K, D) float32
    film_gamma: Optional[np.ndarray] = None  # (B, hidden0) float32
    film_beta: Optional[np.ndarray] = None
    gate: Optional[np.ndarray] = None    # (H, L/2+1) complex64
    reg: Optional[np.ndarray] = None     # (B, R, C) register activations (N-D, registers=R)
    reg_query: Optional[np.ndarray] = None
    film_W: Optional[np.ndarray] = None  # (2 hidden0, C): z(x) -> (gamma, beta)
    film_b: Optional[np.ndarray] = None
    v: Optional[Signal] = None
    xs: list = dataclasses.field(default_factory=list)


def _mlp(rng, widths):
    Ws, bs = [], []
    for l in range(len(widths) - 1):
        bound = 1.0 / math.sqrt(widths[l])
        Ws.append(rng.uniform(-bound, bound, size=(widths[l + 1], widths[l])).astype(np.float32))
        bs.append(rng.uniform(-bound, bound, size=(widths[l + 1],)).astype(np.float32))
    return Ws, bs


def _signal(rng, shape, dtype) -> Signal:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if dtype == "bf16":
        bits = bf16_round(x)
        return Signal(bf16_to_f32(bits), bits)
    return Signal(x)


def spec_of(name: str, **overrides) -> dict:
    spec = dict(WORKLOADS[name])
    spec.update(overrides)
    spec["name"] = name
    return spec


def make(name: str, seed: Optional[int] = None, with_signals: bool = True, **overrides) -> Workload:
    """Draw the inputs of workload ``name`` (shapes may be overridden, e.g.
    smaller B, D or L for tests; the recipe is unchanged)."""
    spec = spec_of(name, **overrides)
    rng = np.random.default_rng(SEEDS.get(name, 0) if seed is None else seed)
    kind = spec["kind"]
    if kind == "operator":
        K = spec["order"] - 1
        width_in = int(spec["include_t"]) + 2 * spec["F"]
        widths = [width_in] + list(spec["hidden"]) + [K * spec["D"]]
        Ws, bs = _mlp(rng, widths)
        lo, hi = spec["alpha"]
        alpha = rng.uniform(lo, hi, size=(K * spec["D"],)).astype(np.float32)
        Dskip = rng.standard_normal(size=(K, spec["D"]), dtype=np.float32) if spec["skip"] else None
        w = Workload(name, spec, Ws, bs, alpha=alpha, Dskip=Dskip)
        if with_signals:
            shape = (spec["B"], spec["D"], spec["L"])
            w.v = _signal(rng, shape, spec["dtype"])
            w.xs = [_signal(rng, shape, spec["dtype"]) for _ in range(K)]
        return w
    if kind == "nd":
        widths = [6 * spec["F"]] + list(spec["hidden"]) + [spec["D"]]
        Ws, bs = _mlp(rng, widths)
        lo, hi = spec["alpha"]
        alpha = rng.uniform(lo, hi, size=(spec["D"],)).astype(np.float32)
        Dskip = rng.standard_normal(size=(1, spec["D"]), dtype=np.float32) if spec["skip"] else None
        gamma = beta = None
        if spec.get("film"):
            gamma = (0.1 * rng.standard_normal(size=(spec["B"], spec["hidden"][0]))).astype(np.float32)
            beta = (0.1 * rng.standard_normal(size=(spec["B"], spec["hidden"][0]))).astype(np.float32)
        w = Workload(name, spec, Ws, bs, alpha=alpha, Dskip=Dskip, film_gamma=gamma, film_beta=beta)
        if with_signals:
            shape = (spec["B"], spec["D"]) + tuple(spec["grid"])
            w.v = _signal(rng, shape, spec["dtype"])
            w.xs = [_signal(rng, shape, spec["dtype"])]
        if spec.get("registers"):
            # input conditioning through register tokens (drawn after everything
            # above, so the draws before stay the same): activations of R
            # registers per sample, the pooling query, and the FiLM map of z(x)
            R, C, H = spec["registers"], spec.get("register_width", 64), spec["hidden"][0]
            w.reg = rng.standard_normal(size=(spec["B"], R, C)).astype(np.float32)
            w.reg_query = (rng.standard_normal(size=(C,)) / math.sqrt(C)).astype(np.float32)
            w.film_W = rng.uniform(-0.1 / math.sqrt(C), 0.1 / math.sqrt(C), size=(2 * H, C)).astype(np.float32)
            w.film_b = (0.01 * rng.standard_normal(size=(2 * H,))).astype(np.float32)
        return w
    if kind == "gate":
        nb = spec["L"] // 2 + 1
        a = rng.standard_normal(size=(spec["H"], nb))
        phi = rng.uniform(-math.pi, math.pi, size=(spec["H"], nb))
        # g = sigmoid(a) * exp(i phi): the workload's fixed, seeded gate (an input)
        gate = ((1.0 / (1.0 + np.exp(-a))) * np.exp(1j * phi)).astype(np.complex64)
        w = Workload(name, spec, [], [], gate=gate)
        if with_signals:
            shape = (spec["B"], spec["H"], spec["Dh"], spec["L"])
            w.v = _signal(rng, shape, spec["dtype"])          # x1 (mixed)
            w.xs = [_signal(rng, shape, spec["dtype"])]       # x2 (output gate)
        return w
    raise ValueError(kind)


def signal_bytes(spec: dict) -> int:
    """Bytes of one input/output signal tensor for a workload."""
    el = 2 if spec["dtype"] == "bf16" else 4
    if spec["kind"] == "operator":
        return spec["B"] * spec["D"] * spec["L"] * el
    if spec["kind"] == "nd":
        return spec["B"] * spec["D"] * int(np.prod(spec["grid"])) * el
    return spec["B"] * spec["H"] * spec["Dh"] * spec["L"] * el
