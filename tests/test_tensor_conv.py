"""The streaming FFT convolution with its radix-32 stages on the tcgen05
tensor cores (bf16 rows of L = 8192, one order; HYENA_FFT_ENGINE=tensor)
against the float64 oracle, next to the fp32 SIMT kernel that is the default
(HYENA_FFT_ENGINE=simt): both engines, gate and skip on and off, guard bands
around the output, more rows than resident CTAs (the persistent row loop and
its prefetch), and repeat calls bit-identical."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import bf16_ulp_diff, check, f32_dev, to_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402

ENGINES = ["tensor", "simt"]


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _filters(rng, D, L):
    t = np.arange(L)
    rate = rng.uniform(0.3, 5.0, size=(D, 1))
    return (rng.standard_normal((D, L)) * np.exp(-rate * t / L)).astype(np.float32)


def _spectra(h32):
    D, L = h32.shape
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(h32), H, rows=D, ndim=1, dims=[L])
    return H


@pytest.mark.parametrize("engine", ENGINES)
def test_operator_rows_vs_direct(engine, monkeypatch):
    monkeypatch.setenv("HYENA_FFT_ENGINE", engine)
    B, D, L = 2, 3, 8192
    w = hw.make("c2", seed=3100, B=B, D=D, L=L)
    h32 = _filters(np.random.default_rng(31), D, L)
    H = _spectra(h32)
    v, x1 = to_dev(w.v, "bf16"), to_dev(w.xs[0], "bf16")
    y = torch.empty_like(v)
    hy.hyena_operator(v, [x1], [H], y, Dskips=[f32_dev(w.Dskip[0])])
    torch.cuda.synchronize()
    ref = oracle.hyena_rows(w.v.f32, [w.xs[0].f32], h32[None].astype(np.float64), w.Dskip)
    check(to_np(y).reshape(B * D, L), ref, "bf16", "%s engine, B2 D3 L8192" % engine)
    assert bf16_ulp_diff(y, ref.reshape(y.shape)) <= 2
    y2 = torch.empty_like(v)
    hy.hyena_operator(v, [x1], [H], y2, Dskips=[f32_dev(w.Dskip[0])])
    assert torch.equal(y, y2)


@pytest.mark.parametrize("engine", ENGINES)
def test_fftconv_variants_and_guard_bands(engine, monkeypatch):
    monkeypatch.setenv("HYENA_FFT_ENGINE", engine)
    B, D, L = 1, 2, 8192
    w = hw.make("c2", seed=3200, B=B, D=D, L=L)
    h32 = _filters(np.random.default_rng(32), D, L)
    H = _spectra(h32)
    u, gate = to_dev(w.v, "bf16"), to_dev(w.xs[0], "bf16")
    dsk = f32_dev(w.Dskip[0])
    n = B * D * L
    for g, s in [(None, None), (gate, None), (None, dsk), (gate, dsk)]:
        buf = torch.full((n + 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
        y = buf[2048:2048 + n].view(B, D, L)
        hy.hyena_fftconv(u, H, y, Dskip=s, gate=g)
        torch.cuda.synchronize()
        assert torch.all(buf[:2048] == 7.0) and torch.all(buf[2048 + n:] == 7.0)
        conv = oracle.hyena_rows(w.v.f32, [np.ones((B, D, L))], h32[None].astype(np.float64),
                                 w.Dskip[:1] if s is not None else None)
        if g is not None:
            conv = conv * w.xs[0].f32.reshape(B * D, L)
        check(to_np(y).reshape(B * D, L), conv, "bf16",
              "%s engine fftconv gate=%s skip=%s" % (engine, g is not None, s is not None))
        assert bf16_ulp_diff(y, conv.reshape(y.shape)) <= 2


def test_more_rows_than_resident_ctas_and_engines_agree(monkeypatch):
    """400 rows (more than two CTAs on each of the 148 SMs): every row against
    the FFT-route reference, 8 against the direct chain; the two engines agree
    to within the bf16 rounding of the output."""
    B, D, L = 4, 100, 8192
    w = hw.make("c2", seed=3300, B=B, D=D, L=L)
    h32 = _filters(np.random.default_rng(33), D, L)
    H = _spectra(h32)
    v, x1 = to_dev(w.v, "bf16"), to_dev(w.xs[0], "bf16")
    outs = {}
    for engine in ENGINES:
        monkeypatch.setenv("HYENA_FFT_ENGINE", engine)
        y = torch.empty_like(v)
        hy.hyena_operator(v, [x1], [H], y, Dskips=[f32_dev(w.Dskip[0])])
        torch.cuda.synchronize()
        outs[engine] = y
    ref = oracle.fft_hyena_rows(w.v.f32, [w.xs[0].f32], h32[None].astype(np.float64), w.Dskip)
    rows = np.random.default_rng(4).choice(B * D, 8, replace=False)
    ref_d = oracle.hyena_rows(w.v.f32, [w.xs[0].f32], h32[None].astype(np.float64), w.Dskip, rows=rows)
    for engine, y in outs.items():
        got = to_np(y).reshape(B * D, L)
        check(got, ref, "bf16", "%s engine, 400 rows (FFT route)" % engine)
        check(got[rows], ref_d, "bf16", "%s engine, 8 rows (direct)" % engine)
        assert bf16_ulp_diff(y, ref.reshape(y.shape)) <= 2
    d = (outs["tensor"].float() - outs["simt"].float()).abs()
    scale = outs["simt"].float().abs().clamp_min(1e-30)
    # the engines differ by at most one bf16 rounding step on all but tiny values
    big = outs["simt"].float().abs() > 1e-2 * outs["simt"].float().pow(2).mean().sqrt()
    assert float((d[big] / scale[big]).max()) <= 2 ** -7
