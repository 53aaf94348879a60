"""Failure detection of the bounded device waits, without a GPU fault.

The self-test makes an mbarrier wait run out (its phase waits for an arrival
that never comes): the kernel records HY_FAULT_SELFTEST and returns, the host
reads the bit (HY_ERR_TIMEOUT from the C call) and the context stays usable.
The streaming convolution, whose row staging waits on mbarriers, then runs
with several rows per persistent CTA, with and without a gate, matches the
oracle on sampled rows and leaves the fault word clear (every GPU test also
checks that word afterwards, in conftest)."""
import ctypes
import time

import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import check, f32_dev, to_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.sets_faults
def test_selftest_wait_runs_out_and_context_survives():
    assert hy.device_faults(clear=True) == 0
    t0 = time.perf_counter()
    hy.selftest_bounded_wait(2000)
    assert hy.device_faults(clear=True) == hy.HY_FAULT_SELFTEST
    assert time.perf_counter() - t0 < 5.0
    assert hy.device_faults(clear=True) == 0
    # the C status of a set word, then a clear that sticks
    hy.selftest_bounded_wait(500)
    v = ctypes.c_uint32(0)
    st = hy.lib().hyena_device_faults(ctypes.byref(v), 1, torch.cuda.current_stream().cuda_stream)
    assert st == 5 and v.value == hy.HY_FAULT_SELFTEST
    assert b"gave up" in hy.lib().hyena_last_error()
    st = hy.lib().hyena_device_faults(ctypes.byref(v), 0, torch.cuda.current_stream().cuda_stream)
    assert st == 0 and v.value == 0
    # the context still runs kernels correctly
    a = torch.arange(1 << 20, device="cuda", dtype=torch.float32)
    assert float(a.sum()) == float((1 << 20) * ((1 << 20) - 1) // 2)


@pytest.mark.parametrize("dtype,gate", [("f32", True), ("f32", False), ("bf16", True), ("bf16", False)])
def test_stream_rows_per_cta(dtype, gate):
    """B2 D320 L8192: 640 rows on at most 2 x 148 persistent CTAs, so every
    CTA re-arms its barriers for several rows."""
    B, D, L = 2, 320, 8192
    w = hw.make("c1", seed=4242, B=B, D=D, L=L, dtype=dtype)
    rng = np.random.default_rng(9)
    t = np.arange(L)
    h32 = (rng.standard_normal((1, D, L)) * np.exp(-rng.uniform(0.5, 4.0, (1, D, 1)) * t / L)).astype(np.float32)
    H = torch.empty((D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(h32[0]), H, rows=D, ndim=1, dims=[L])
    u = to_dev(w.v, dtype)
    g = to_dev(w.xs[0], dtype) if gate else None
    dsk = f32_dev(w.Dskip[0])
    y = torch.empty_like(u)
    hy.hyena_fftconv(u, H, y, Dskip=dsk, gate=g)
    assert hy.device_faults(clear=False) == 0
    rows = np.random.default_rng(3).choice(B * D, 12, replace=False)
    xs = [w.xs[0].f32 if gate else np.ones((B, D, L))]
    ref = oracle.hyena_rows(w.v.f32, xs, h32.astype(np.float64), w.Dskip[:1], rows=rows)
    check(to_np(y).reshape(B * D, L)[rows], ref, dtype, "stream B%d D%d L%d %s gate=%s" % (B, D, L, dtype, gate))
