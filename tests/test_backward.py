"""Backward pass of the operator against the float64 oracle (explicit
adjoint matrices, pinned to finite differences of the direct forward):
orders 2 to 4, fp32 and bf16 I/O, ragged lengths, with and without the
skip term, gradients of the inputs, the gates, the filters and D; one
multi-pass length; the fused order-2 kernel (power-of-two rows) at small
sizes in full and at the 8192-sample width on sampled indices."""
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


def _spectra(h32):
    K, D, L = h32.shape
    H = torch.empty((K * D, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    wsb = hy.filter_spectrum_workspace(K * D, 1, [L])
    hy.hyena_filter_spectrum(f32_dev(h32.reshape(K * D, L)), H, rows=K * D, ndim=1, dims=[L],
                             ws=torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda"))
    return [H[k * D:(k + 1) * D] for k in range(K)]


@pytest.mark.parametrize("B,D,L,order,dtype,skip", [
    (2, 3, 1000, 2, "f32", True),
    (1, 4, 777, 3, "f32", False),
    (3, 2, 2048, 2, "bf16", True),
    (1, 2, 300, 4, "f32", True),
    # order 2 over power-of-two rows: the fused per-channel kernel
    (4, 3, 512, 2, "f32", True),
    (2, 3, 1024, 2, "bf16", False),
    (5, 2, 2048, 2, "f32", True),
    (1, 1, 4096, 2, "f32", True),
])
def test_backward_vs_oracle(B, D, L, order, dtype, skip):
    K = order - 1
    rng = np.random.default_rng(L + 10 * order)
    t = np.arange(L)
    h = (rng.standard_normal((K, D, L)) * np.exp(-rng.uniform(0.5, 3.0, (K, D, 1)) * t / L)).astype(np.float32)
    Dk = rng.standard_normal((K, D)).astype(np.float32) if skip else None
    sig = lambda: hw.Signal(rng.standard_normal((B, D, L)).astype(np.float32))
    v, dy = sig(), sig()
    xs = [sig() for _ in range(K)]
    if dtype == "bf16":
        for s_ in [v, dy] + xs:
            s_.bf16 = hw.bf16_round(s_.f32)
            s_.f32 = hw.bf16_to_f32(s_.bf16)
    Hs = _spectra(h)
    vd, dyd = to_dev(v, dtype), to_dev(dy, dtype)
    xd = [to_dev(x, dtype) for x in xs]
    dv = torch.empty_like(vd)
    dxs = [torch.empty_like(vd) for _ in range(K)]
    dhs = [torch.empty((D, L), device="cuda") for _ in range(K)]
    dDs = [torch.empty(D, device="cuda") for _ in range(K)]
    code = hy.HY_BF16 if dtype == "bf16" else hy.HY_F32
    ws = torch.empty(hy.operator_backward_workspace(order, B, D, L, code), dtype=torch.uint8, device="cuda")
    hy.hyena_operator_backward(vd, xd, Hs, dyd, dv, dxs, Dskips=[f32_dev(Dk[k]) for k in range(K)] if skip else None,
                               dhs=dhs, dDs=dDs, ws=ws)
    torch.cuda.synchronize()
    rdv, rdx, rdh, rdD = oracle.hyena_backward(v.f32, [x.f32 for x in xs], h, Dk, dy.f32)
    check(to_np(dv), rdv, dtype, "dv")
    for k in range(K):
        check(to_np(dxs[k]), rdx[k], dtype, "dx_%d" % k)
        # filter and skip gradients are fp32 sums; their tolerance follows the I/O precision of the inputs
        check(to_np(dhs[k]), rdh[k], "f32", "dh_%d" % k)
        check(to_np(dDs[k]), rdD[k], "f32", "dD_%d" % k)


def test_backward_optional_outputs_and_reuse():
    """dh / dD may be omitted; the result for dv and dx does not change, and a
    second call on the same workspace repeats it bit for bit."""
    B, D, L, order = 2, 2, 512, 3
    rng = np.random.default_rng(3)
    h = (rng.standard_normal((2, D, L)) * 0.1).astype(np.float32)
    Hs = _spectra(h)
    v, dy = (f32_dev(rng.standard_normal((B, D, L)).astype(np.float32)) for _ in range(2))
    xs = [f32_dev(rng.standard_normal((B, D, L)).astype(np.float32)) for _ in range(2)]
    ws = torch.empty(hy.operator_backward_workspace(order, B, D, L, hy.HY_F32), dtype=torch.uint8, device="cuda")
    outs = []
    for with_extra in (True, False, False):
        dv = torch.empty_like(v)
        dxs = [torch.empty_like(v) for _ in range(2)]
        extra = dict(dhs=[torch.empty((D, L), device="cuda") for _ in range(2)], dDs=[None, torch.empty(D, device="cuda")]) \
            if with_extra else {}
        hy.hyena_operator_backward(v, xs, Hs, dy, dv, dxs, ws=ws, **extra)
        torch.cuda.synchronize()
        outs.append([dv.clone()] + [d.clone() for d in dxs])
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)
    for a, b in zip(outs[1], outs[2]):
        assert torch.equal(a, b)


def test_backward_multipass_length_sampled():
    """L = 20000 runs every convolution of the backward on the multi-pass
    path; checked against the direct sums at 97 sampled indices and lags
    (with the full-row RMS as the scale) and dD in full."""
    from _helpers import check_part
    B, D, L = 2, 2, 20000
    rng = np.random.default_rng(7)
    t = np.arange(L)
    h = (rng.standard_normal((1, D, L)) * np.exp(-rng.uniform(0.5, 3.0, (1, D, 1)) * t / L)).astype(np.float32)
    Dk = rng.standard_normal((1, D)).astype(np.float32)
    v, x1, dy = (rng.standard_normal((B, D, L)).astype(np.float32) for _ in range(3))
    Hs = _spectra(h)
    dv = torch.empty((B, D, L), device="cuda")
    dx = [torch.empty_like(dv)]
    dh = [torch.empty((D, L), device="cuda")]
    dD = [torch.empty(D, device="cuda")]
    ws = torch.empty(hy.operator_backward_workspace(2, B, D, L, hy.HY_F32), dtype=torch.uint8, device="cuda")
    hy.hyena_operator_backward(f32_dev(v), [f32_dev(x1)], Hs, f32_dev(dy), dv, dx, Dskips=[f32_dev(Dk[0])],
                               dhs=dh, dDs=dD, ws=ws)
    torch.cuda.synchronize()
    ts = np.unique(np.concatenate([[0, 1, L // 2, L - 2, L - 1], rng.choice(L, 92, replace=False)]))
    sv, sx, sh, sD = oracle.hyena_backward_samples(v, x1, h[0], Dk[0], dy, ts)
    gdv, gdx, gdh = to_np(dv), to_np(dx[0]), to_np(dh[0])
    rms = lambda a: float(np.sqrt(np.mean(a.astype(np.float64) ** 2)))
    check_part(gdv[..., ts], sv, rms(gdv), "f32", "dv L=20000")
    check_part(gdx[..., ts], sx, rms(gdx), "f32", "dx L=20000")
    check_part(gdh[:, ts], sh, rms(gdh), "f32", "dh L=20000")
    check(to_np(dD[0]), sD, "f32", "dD L=20000")


def test_backward_fused_width_8192_sampled():
    """Order 2, bf16, L = 8192 (the fused kernel at the widest row it takes,
    with eight samples per channel summed into dh and dD): direct sums at 40
    indices and lags of every row, dD in full."""
    from _helpers import check_part
    B, D, L = 8, 6, 8192
    rng = np.random.default_rng(11)
    t = np.arange(L)
    h = (rng.standard_normal((1, D, L)) * np.exp(-rng.uniform(0.5, 3.0, (1, D, 1)) * t / L)).astype(np.float32)
    Dk = rng.standard_normal((1, D)).astype(np.float32)
    sig = lambda: hw.Signal(rng.standard_normal((B, D, L)).astype(np.float32))
    v, x1, dy = sig(), sig(), sig()
    for s_ in (v, x1, dy):
        s_.bf16 = hw.bf16_round(s_.f32)
        s_.f32 = hw.bf16_to_f32(s_.bf16)
    Hs = _spectra(h)
    vd, xd, dyd = (to_dev(a, "bf16") for a in (v, x1, dy))
    dv = torch.empty_like(vd)
    dx = [torch.empty_like(vd)]
    dh = [torch.empty((D, L), device="cuda")]
    dD = [torch.empty(D, device="cuda")]
    ws = torch.empty(hy.operator_backward_workspace(2, B, D, L, hy.HY_BF16), dtype=torch.uint8, device="cuda")
    hy.hyena_operator_backward(vd, [xd], Hs, dyd, dv, dx, Dskips=[f32_dev(Dk[0])], dhs=dh, dDs=dD, ws=ws)
    torch.cuda.synchronize()
    ts = np.unique(np.concatenate([[0, 1, L // 2, L - 2, L - 1], rng.choice(L, 35, replace=False)]))
    sv, sx, sh, sD = oracle.hyena_backward_samples(v.f32, x1.f32, h[0], Dk[0], dy.f32, ts)
    gdv, gdx, gdh = to_np(dv), to_np(dx[0]), to_np(dh[0])
    rms = lambda a: float(np.sqrt(np.mean(a.astype(np.float64) ** 2)))
    check_part(gdv[..., ts], sv, rms(gdv), "bf16", "dv L=8192")
    check_part(gdx[..., ts], sx, rms(gdx), "bf16", "dx L=8192")
    check_part(gdh[:, ts], sh, rms(gdh), "f32", "dh L=8192")
    check(to_np(dD[0]), sD, "f32", "dD L=8192")


def test_backward_fused_optional_outputs_and_reuse():
    """Order 2 on the fused kernel: dh and dD may each be omitted without
    changing dv and dx, a repeated call is bit-identical (no atomics), and
    with dh alone its lag-0 value is dD."""
    B, D, L = 3, 4, 1024
    rng = np.random.default_rng(5)
    h = (rng.standard_normal((1, D, L)) * 0.05).astype(np.float32)
    Hs = _spectra(h)
    v, x1, dy = (f32_dev(rng.standard_normal((B, D, L)).astype(np.float32)) for _ in range(3))
    Dk = [f32_dev(rng.standard_normal(D).astype(np.float32))]
    ws = torch.empty(hy.operator_backward_workspace(2, B, D, L, hy.HY_F32), dtype=torch.uint8, device="cuda")
    outs = []
    for extra in ({"dhs": [torch.empty((D, L), device="cuda")], "dDs": [torch.empty(D, device="cuda")]},
                  {"dhs": [torch.empty((D, L), device="cuda")]}, {"dDs": [torch.empty(D, device="cuda")]}, {},
                  {"dhs": [torch.empty((D, L), device="cuda")], "dDs": [torch.empty(D, device="cuda")]}):
        dv = torch.empty_like(v)
        dx = [torch.empty_like(v)]
        hy.hyena_operator_backward(v, [x1], Hs, dy, dv, dx, Dskips=Dk, ws=ws, **extra)
        torch.cuda.synchronize()
        outs.append((dv.clone(), dx[0].clone(), extra))
    for dv, dx, _ in outs[1:]:
        assert torch.equal(dv, outs[0][0]) and torch.equal(dx, outs[0][1])
    a, b = outs[0][2], outs[4][2]
    assert torch.equal(a["dhs"][0], b["dhs"][0]) and torch.equal(a["dDs"][0], b["dDs"][0])
    assert torch.equal(outs[1][2]["dhs"][0], a["dhs"][0])
    assert torch.equal(outs[2][2]["dDs"][0], a["dDs"][0])
    lag0 = to_np(a["dhs"][0])[:, 0].astype(np.float64)
    dd = to_np(a["dDs"][0]).astype(np.float64)
    assert np.max(np.abs(lag0 - dd)) <= 1e-4 * np.sqrt(np.mean(dd ** 2))


def test_backward_fused_channels_shared_by_two_ctas():
    """Order 2, fp32, L = 8192 with more channels than CTAs (600 rows over
    the SMs): a channel's rows are split between two CTAs whose partial dh and
    dD meet in the output; checked against direct sums at sampled indices and
    lags of every channel, dD in full, and a repeated call bit for bit."""
    from _helpers import check_part
    B, D, L = 3, 200, 8192
    rng = np.random.default_rng(21)
    t = np.arange(L)
    h = (rng.standard_normal((1, D, L)) * np.exp(-rng.uniform(0.5, 3.0, (1, D, 1)) * t / L)).astype(np.float32)
    Dk = rng.standard_normal((1, D)).astype(np.float32)
    v, x1, dy = (rng.standard_normal((B, D, L)).astype(np.float32) for _ in range(3))
    Hs = _spectra(h)
    ws = torch.empty(hy.operator_backward_workspace(2, B, D, L, hy.HY_F32), dtype=torch.uint8, device="cuda")
    res = []
    for _ in range(2):
        dv = torch.empty((B, D, L), device="cuda")
        dx = [torch.empty_like(dv)]
        dh = [torch.empty((D, L), device="cuda")]
        dD = [torch.empty(D, device="cuda")]
        hy.hyena_operator_backward(f32_dev(v), [f32_dev(x1)], Hs, f32_dev(dy), dv, dx, Dskips=[f32_dev(Dk[0])],
                                   dhs=dh, dDs=dD, ws=ws)
        torch.cuda.synchronize()
        res.append((dv, dx[0], dh[0], dD[0]))
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)
    ts = np.unique(np.concatenate([[0, 1, L - 1], rng.choice(L, 9, replace=False)]))
    sv, sx, sh, sD = oracle.hyena_backward_samples(v, x1, h[0], Dk[0], dy, ts)
    gdv, gdx, gdh = (to_np(a) for a in res[0][:3])
    rms = lambda a: float(np.sqrt(np.mean(a.astype(np.float64) ** 2)))
    check_part(gdv[..., ts], sv, rms(gdv), "f32", "dv")
    check_part(gdx[..., ts], sx, rms(gdx), "f32", "dx")
    check_part(gdh[:, ts], sh, rms(gdh), "f32", "dh")
    check(to_np(res[0][3]), sD, "f32", "dD")
