"""Parity of the single-launch (on-chip) path against the float64 oracle:
filter generator, filter spectrum, gated convolution chain and spectral gate,
on seeded inputs, across sizes that span several FFT stages, ragged lengths,
odd batch/channel counts, the degenerate L = 1, and the full-size workloads
(sampled rows checked by the direct O(L^2) definition, all rows by the
FFT-route reference that the CPU tests pin to it)."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import (bf16_ulp_diff, c64_dev, check, f32_dev, rel_l2, to_dev, to_np)

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _decaying_filters(rng, K, D, L):
    t = np.arange(L)
    rate = rng.uniform(0.5, 4.0, size=(K, D, 1))
    return (rng.standard_normal((K, D, L)) * np.exp(-rate * t / max(L, 1))).astype(np.float32)


def gpu_spectra(h32):
    """(K, D, L) float32 -> list of K device spectra (D, bins) via the library."""
    K, D, L = h32.shape
    nb = hy.spectrum_bins(L)
    hd = f32_dev(h32.reshape(K * D, L))
    H = torch.empty((K * D, nb), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(hd, H, rows=K * D, ndim=1, dims=[L])
    return [H[k * D:(k + 1) * D] for k in range(K)], H


CASES = [
    # B, D, L, order, dtype, skip
    (1, 3, 16, 2, "f32", True),
    (3, 2, 1, 2, "f32", True),
    (1, 1, 17, 2, "f32", False),
    (2, 5, 100, 2, "f32", True),
    (2, 3, 64, 4, "f32", True),
    (1, 4, 1000, 3, "bf16", True),
    (2, 3, 777, 2, "bf16", True),
    (1, 2, 2048, 2, "f32", True),
    (1, 2, 4096, 2, "bf16", False),
    (3, 2, 8192, 2, "f32", True),
    (1, 3, 8192, 3, "f32", True),
    (1, 2, 16384, 2, "f32", True),
    (1, 2, 16000, 3, "bf16", True),
]


@pytest.mark.parametrize("B,D,L,order,dtype,skip", CASES)
def test_operator_vs_oracle(B, D, L, order, dtype, skip):
    w = hw.make("c3", seed=1000 + L + order, B=B, D=D, L=L, order=order, dtype=dtype, skip=skip)
    rng = np.random.default_rng(L * 7 + D)
    K = order - 1
    h32 = _decaying_filters(rng, K, D, L)
    Hs, H = gpu_spectra(h32)
    # the spectra themselves against the (pinned) FFT-route reference
    Href = oracle.fft_spectrum(h32.reshape(K * D, L), n=2 * (hy.spectrum_bins(L) - 1))
    Hgot = H.cpu().numpy().astype(np.complex128)
    check(np.stack([Hgot.real, Hgot.imag]), np.stack([Href.real, Href.imag]), "f32", "spectrum")
    v = to_dev(w.v, dtype)
    xs = [to_dev(x, dtype) for x in w.xs]
    y = torch.empty_like(v)
    dsk = [f32_dev(w.Dskip[k]) for k in range(K)] if skip else None
    hy.hyena_operator(v, xs, Hs, y, Dskips=dsk)
    torch.cuda.synchronize()
    ref = oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], h32.astype(np.float64),
                            w.Dskip if skip else None)
    got = to_np(y).reshape(B * D, L)
    check(got, ref, dtype, "operator B%d D%d L%d order%d" % (B, D, L, order))
    if dtype == "bf16":
        assert bf16_ulp_diff(y, ref.reshape(y.shape)) <= 2
    # a second call is bit-identical
    y2 = torch.empty_like(v)
    hy.hyena_operator(v, xs, Hs, y2, Dskips=dsk)
    assert torch.equal(y, y2)


def test_fftconv_gate_skip_variants_and_guard_bands():
    B, D, L = 2, 3, 512
    w = hw.make("c1", seed=77, B=B, D=D, L=L)
    rng = np.random.default_rng(5)
    h32 = _decaying_filters(rng, 1, D, L)
    Hs, _ = gpu_spectra(h32)
    u = to_dev(w.v, "f32")
    gate = to_dev(w.xs[0], "f32")
    dsk = f32_dev(w.Dskip[0])
    n = B * D * L
    for g, s in [(None, None), (gate, None), (None, dsk), (gate, dsk)]:
        buf = torch.full((n + 2048,), 12345.0, device="cuda")
        y = buf[1024:1024 + n].view(B, D, L)
        hy.hyena_fftconv(u, Hs[0], y, Dskip=s, gate=g)
        torch.cuda.synchronize()
        assert torch.all(buf[:1024] == 12345.0) and torch.all(buf[1024 + n:] == 12345.0)
        conv = oracle.hyena_rows(w.v.f32, [np.ones((B, D, L))], h32.astype(np.float64),
                                 w.Dskip[:1] if s is not None else None)
        if g is not None:
            conv = conv * w.xs[0].f32.reshape(B * D, L)
        check(to_np(y).reshape(B * D, L), conv, "f32", "fftconv gate=%s skip=%s" % (g is not None, s is not None))


@pytest.mark.parametrize("engine", ["default", "simt"])
def test_filter_gen_1d_vs_oracle(engine, monkeypatch):
    """The filters of workloads 1-3 (c3 at L = 4096) with the default engine
    choice and with HYENA_FILTER_ENGINE=simt (FP32-pipe kernels).  These
    lengths have fewer 128-position tiles than SMs: by default workload 2's
    three layers and 768 outputs run all on the tensor cores (one CTA per
    tile and slice group); the others run the streaming kernel."""
    if engine == "simt":
        monkeypatch.setenv("HYENA_FILTER_ENGINE", "simt")
    for name, L in [("c1", 1024), ("c2", 8192), ("c3", 4096)]:
        w = hw.make(name, with_signals=False, L=L)
        spec = w.spec
        h = torch.empty((w.Ws[-1].shape[0], L), device="cuda")
        hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                            alpha=f32_dev(w.alpha), n_freq=spec["F"], include_t=spec["include_t"])
        torch.cuda.synchronize()
        ref = oracle.filter_gen_1d(L, spec["F"], spec["include_t"], w.Ws, w.bs, w.alpha)
        check(to_np(h), ref, "f32", "filter_gen %s" % name)


def _mlp(rng, widths):
    Ws, bs = [], []
    for a, b in zip(widths[:-1], widths[1:]):
        lim = 1.0 / np.sqrt(a)
        Ws.append(rng.uniform(-lim, lim, (b, a)).astype(np.float32))
        bs.append(rng.uniform(-lim, lim, b).astype(np.float32))
    return Ws, bs


@pytest.mark.parametrize("L,F,include_t,hidden,nout,offset", [
    (1, 2, True, [8], 3, 0),                 # one position
    (777, 3, True, [33], 130, 0),            # ragged length, odd widths, two last-layer tiles
    (1000, 5, False, [100, 20, 7], 300, 1),  # four layers, misaligned output rows
    (4096, 16, True, [], 64, 0),             # single layer (encoding -> output)
    (3000, 64, True, [128], 40, 0),          # widest encoding (129) and hidden (128)
])
def test_filter_gen_1d_shapes(L, F, include_t, hidden, nout, offset):
    rng = np.random.default_rng(L + nout)
    w0 = int(include_t) + 2 * F
    Ws, bs = _mlp(rng, [w0] + hidden + [nout])
    alpha = rng.uniform(0.1, 4.0, nout).astype(np.float32)
    flat = torch.full((nout * L + offset,), float("nan"), device="cuda")
    h = flat[offset:].view(nout, L)
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=include_t)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, include_t, Ws, bs, alpha)
    check(to_np(h), ref, "f32", "filter_gen L%d widths %s" % (L, [w0] + hidden + [nout]))
    if offset:
        assert np.isnan(to_np(flat[:offset])).all()


@pytest.mark.parametrize("act,window", [("sine", "gauss"), ("identity", "exp"), ("sine", "exp")])
def test_filter_gen_1d_activations_and_windows(act, window):
    rng = np.random.default_rng(41)
    L, F, nout = 3000, 8, 150
    widths = [1 + 2 * F, 48, 40, nout]
    Ws, bs = _mlp(rng, widths)
    omega = rng.uniform(0.5, 8, 88).astype(np.float32) if act == "sine" else None
    alpha = rng.uniform(0.2, 5.0, nout).astype(np.float32)
    h = torch.empty((nout, L), device="cuda")
    codes = {"silu": hy.HY_ACT_SILU, "identity": hy.HY_ACT_IDENTITY, "sine": hy.HY_ACT_SINE}
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=True, act=codes[act],
                        omega=f32_dev(omega) if omega is not None else None,
                        window=hy.HY_WIN_GAUSS if window == "gauss" else hy.HY_WIN_EXP)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act=act, omega=omega, window=window)
    check(to_np(h), ref, "f32", "filter_gen %s/%s" % (act, window))


def test_c1_end_to_end():
    """Workload 1 exactly: MLP parameters -> filters -> spectra -> operator."""
    w = hw.make("c1")
    s = w.spec
    B, D, L = s["B"], s["D"], s["L"]
    h = torch.empty((D, L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=s["F"], include_t=True)
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(h, H, rows=D, ndim=1, dims=[L])
    v, x1 = to_dev(w.v, "f32"), to_dev(w.xs[0], "f32")
    y = torch.empty_like(v)
    hy.hyena_operator(v, [x1], [H], y, Dskips=[f32_dev(w.Dskip[0])])
    torch.cuda.synchronize()
    h64 = oracle.filter_gen_1d(L, s["F"], True, w.Ws, w.bs, w.alpha)
    ref = oracle.hyena_rows(w.v.f32, [w.xs[0].f32], h64.reshape(1, D, L), w.Dskip)
    check(to_np(y).reshape(B * D, L), ref, "f32", "c1 end-to-end")


@pytest.mark.parametrize("engine", ["tensor", "simt"])
def test_c2_full_size(engine, monkeypatch):
    """Workload 2 at full size (B8 D768 L8192, bf16 I/O) in the launch the
    benchmark times, with the radix-32 FFT stages on the fp32 SIMT pipes (the
    default) and on the tensor cores: all rows against the FFT-route
    reference, 16 sampled rows against the direct O(L^2) chain."""
    monkeypatch.setenv("HYENA_FFT_ENGINE", engine)
    w = hw.make("c2")
    s = w.spec
    B, D, L = s["B"], s["D"], s["L"]
    h = torch.empty((D, L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=s["F"], include_t=True)
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(h, H, rows=D, ndim=1, dims=[L])
    v, x1 = to_dev(w.v, "bf16"), to_dev(w.xs[0], "bf16")
    y = torch.empty_like(v)
    hy.hyena_operator(v, [x1], [H], y, Dskips=[f32_dev(w.Dskip[0])])
    torch.cuda.synchronize()
    h64 = oracle.filter_gen_1d(L, s["F"], True, w.Ws, w.bs, w.alpha)
    check(to_np(h), h64, "f32", "c2 filters")
    got = to_np(y).reshape(B * D, L)
    rows = np.random.default_rng(2).choice(B * D, 16, replace=False)
    ref_rows = oracle.hyena_rows(w.v.f32, [w.xs[0].f32], h64.reshape(1, D, L), w.Dskip, rows=rows)
    check(got[rows], ref_rows, "bf16", "c2 sampled rows (direct), %s engine" % engine)
    ref_all = oracle.fft_hyena_rows(w.v.f32, [w.xs[0].f32], h64.reshape(1, D, L), w.Dskip)
    r = check(got, ref_all, "bf16", "c2 all rows (FFT route), %s engine" % engine)
    assert r < 5e-3
    assert bf16_ulp_diff(y, ref_all.reshape(y.shape)) <= 2


GATE_CASES = [
    # B, H, Dh, L, dtype, x2, shared
    (1, 1, 1, 32, "f32", True, True),
    (2, 3, 2, 64, "f32", True, False),
    (1, 2, 3, 1024, "f32", False, True),
    (2, 2, 2, 4096, "bf16", True, False),
    (1, 2, 2, 32768, "f32", True, True),
]


@pytest.mark.parametrize("B,Hh,Dh,L,dtype,use_x2,shared", GATE_CASES)
def test_spectral_gate_vs_oracle(B, Hh, Dh, L, dtype, use_x2, shared):
    # per-sample gates: draw B*Hh gate rows (sample b uses rows b*Hh..), keep Hh heads of signal
    w = hw.make("c5", seed=900 + L, B=B, H=Hh if shared else Hh * B, Dh=Dh, L=L, dtype=dtype)

    def heads(sig):
        return hw.Signal(np.ascontiguousarray(sig.f32[:, :Hh]),
                         None if sig.bf16 is None else np.ascontiguousarray(sig.bf16[:, :Hh]))
    x1, x2 = heads(w.v), heads(w.xs[0])
    xd = to_dev(x1, dtype)
    x2d = to_dev(x2, dtype) if use_x2 else None
    g = c64_dev(w.gate)
    y = torch.empty_like(xd)
    stride = 0 if shared else Hh * (L // 2 + 1)
    hy.spectral_gate(xd, g, y, x2=x2d, g_batch_stride=stride)
    torch.cuda.synchronize()
    nb = L // 2 + 1
    R = B * Hh * Dh
    kidx = np.array([(0 if shared else b * Hh) + h for b in range(B) for h in range(Hh) for _ in range(Dh)])
    gates = w.gate.astype(np.complex128)
    x1r = x1.f32.reshape(R, L)
    x2r = x2.f32.reshape(R, L) if use_x2 else None
    ref = oracle.fft_spectral_gate_rows(gates[kidx], x1r, x2r)
    got = to_np(y).reshape(R, L)
    check(got, ref, dtype, "spectral gate L%d" % L)
    if L <= 4096:
        kap = np.stack([oracle.gate_kernel(gg) for gg in gates])
        sel = np.arange(min(R, 4))
        direct = oracle.circular_conv_rows(kap, kidx[sel], x1r[sel], None if x2r is None else x2r[sel])
        check(got[sel], direct, dtype, "spectral gate direct L%d" % L)


def test_c5_full_size():
    """Workload 5 at full size (B4 H32 Dh64 L32768 bf16): all rows against the
    FFT-route reference, 6 rows against the direct circular definition."""
    w = hw.make("c5")
    s = w.spec
    B, Hh, Dh, L = s["B"], s["H"], s["Dh"], s["L"]
    xd, x2d = to_dev(w.v, "bf16"), to_dev(w.xs[0], "bf16")
    y = torch.empty_like(xd)
    hy.spectral_gate(xd, c64_dev(w.gate), y, x2=x2d)
    torch.cuda.synchronize()
    R = B * Hh * Dh
    kidx = np.tile(np.repeat(np.arange(Hh), Dh), B)
    got = to_np(y).reshape(R, L)
    ref = oracle.fft_spectral_gate_rows(w.gate.astype(np.complex128)[kidx], w.v.f32.reshape(R, L),
                                        w.xs[0].f32.reshape(R, L))
    check(got, ref, "bf16", "c5 all rows (FFT route)")
    rows = np.array([0, 1, 777, 4095, 6000, R - 1])
    kap = {int(h): oracle.gate_kernel(w.gate[h].astype(np.complex128)) for h in set(kidx[rows])}
    hs = sorted(kap)
    direct = oracle.circular_conv_rows(np.stack([kap[h] for h in hs]), [hs.index(int(k)) for k in kidx[rows]],
                                       w.v.f32.reshape(R, L)[rows], w.xs[0].f32.reshape(R, L)[rows])
    check(got[rows], direct, "bf16", "c5 sampled rows (direct)")
    assert rel_l2(got, ref) < 5e-3


@pytest.mark.parametrize("engine", ["simt", "tensor", "tensor_last"])
@pytest.mark.parametrize("act,hidden,nout", [("silu", [32, 24], 40), ("sine", [32, 24], 40),
                                               ("silu", [96], 200), ("silu", [64], 512),
                                               ("sine", [64], 40), ("silu", [40], 200)])
def test_filter_gen_resident_weights_many_tiles(act, hidden, nout, engine, monkeypatch):
    """Enough positions for the persistent filter kernels: with one hidden
    layer of <= 64 units both layers on the tensor cores (the default; the
    encoding written straight into the first MMA operand, hidden units read
    back from tensor memory, output slices of <= 128), else the last layer
    alone (HYENA_FILTER_ENGINE=tensor_last forces that kernel: 128-position
    tiles as the MMA M, fp16 hi/lo operands, fp32 accumulation) or, with
    HYENA_FILTER_ENGINE=simt, the FP32 pipes with resident weights (or the
    streaming kernel when they do not fit two CTAs per SM): 1-D L = 2^17, one
    or two hidden layers of 24 to 96 units (padded to 16, one or two 64-element
    atoms) and 40, 200 or 512 outputs (one MMA N chunk or several, one output
    slice or several, the last one ragged); every position and output against
    the oracle."""
    monkeypatch.setenv("HYENA_FILTER_ENGINE", engine)
    L, F = 1 << 17, 8
    rng = np.random.default_rng(170 + (act == "sine") + nout)
    widths = [1 + 2 * F] + hidden + [nout]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.1, 2.0, widths[-1]).astype(np.float32)
    omega = rng.uniform(1, 4, sum(hidden)).astype(np.float32) if act == "sine" else None
    h = torch.empty((widths[-1], L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=True,
                        act=hy.HY_ACT_SINE if act == "sine" else hy.HY_ACT_SILU,
                        omega=f32_dev(omega) if omega is not None else None)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act=act, omega=omega)
    check(to_np(h), ref, "f32", "resident-weight filters L=2^17 (%s, %s)" % (act, engine))


@pytest.mark.parametrize("act", ["silu", "sine"])
def test_filter_gen_two_layers_length_not_power_of_two(act):
    """Both layers on the tensor cores with L = 3 * 2^14 (the encoding's
    phase j t mod L by an integer remainder rather than a mask), a ragged
    last tile of positions and 72 outputs; every position and output against
    the oracle."""
    L, F = 3 * (1 << 14) + 77, 6
    rng = np.random.default_rng(4915 + (act == "sine"))
    widths = [1 + 2 * F, 48, 72]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.1, 2.0, widths[-1]).astype(np.float32)
    omega = rng.uniform(1, 4, widths[1]).astype(np.float32) if act == "sine" else None
    h = torch.empty((widths[-1], L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=True,
                        act=hy.HY_ACT_SINE if act == "sine" else hy.HY_ACT_SILU,
                        omega=f32_dev(omega) if omega is not None else None)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act=act, omega=omega)
    check(to_np(h), ref, "f32", "two-layer filters L=%d (%s)" % (L, act))


@pytest.mark.parametrize("act", ["silu", "sine"])
def test_filter_gen_three_layers_few_tiles(act):
    """Two hidden layers and many outputs over fewer 128-position tiles than
    SMs (L = 5000: 40 tiles; 600 outputs): all three layers on the tensor
    cores, each CTA one tile and a group of 128-output slices (grid z = 3:
    slices 0, 3 / 1, 4 / 2, the last one ragged at 88 outputs); an 81-wide
    encoding (two 64-column operand atoms), hidden widths 48 and 40 (padded
    to 48), SiLU or SIREN; every position and output against the oracle."""
    L, F = 5000, 40
    rng = np.random.default_rng(5003 + (act == "sine"))
    widths = [1 + 2 * F, 48, 40, 600]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.1, 2.0, widths[-1]).astype(np.float32)
    omega = rng.uniform(1, 3, 48 + 40).astype(np.float32) if act == "sine" else None
    h = torch.empty((widths[-1], L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=True,
                        act=hy.HY_ACT_SINE if act == "sine" else hy.HY_ACT_SILU,
                        omega=f32_dev(omega) if omega is not None else None)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act=act, omega=omega)
    check(to_np(h), ref, "f32", "three-layer filters L=5000 (%s)" % act)


@pytest.mark.parametrize("engine", ["default", "simt", "tensor_last"])
def test_filter_gen_output_slices(engine, monkeypatch):
    """600 outputs with enough positions, split over grid z: by default both
    layers on the tensor cores in 128-output slices (4 x 128 + 88), with
    HYENA_FILTER_ENGINE=tensor_last the last layer alone in 256-output slices
    (256 + 256 + 88, the last slice padded to 96 MMA columns); L = 2^16, every
    position and output against the oracle.  "simt" runs the FP32-pipe
    kernels on the same filters."""
    if engine != "default":
        monkeypatch.setenv("HYENA_FILTER_ENGINE", engine)
    L, F = 1 << 16, 8
    rng = np.random.default_rng(600)
    widths = [1 + 2 * F, 64, 600]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.1, 2.0, widths[-1]).astype(np.float32)
    h = torch.empty((widths[-1], L), device="cuda")
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, include_t=True)
    torch.cuda.synchronize()
    ref = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha)
    check(to_np(h), ref, "f32", "filters with 600 outputs (%s)" % engine)
