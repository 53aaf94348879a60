"""Parity of the HyenaND 3-D path (filter generator on the grid, 3-D filter
spectrum, gated global convolution) against the float64 oracle: tiny grids on
every voxel by the direct definition, shared and per-sample kernels, circular
and zero-padded boundaries, skip and gate, and workload 4 at full size
(B2 D128 64^3, FiLM-conditioned filters)."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import c64_dev, check, check_part, f32_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def gpu_spectrum3(Kern, circular=False):
    """(R, S, S, S) float32 kernels -> device (R, S, S, S/2+1) via the library."""
    R, S = Kern.shape[0], Kern.shape[1]
    H = torch.empty((R, S, S, S // 2 + 1), dtype=torch.complex64, device="cuda")
    g = S if circular else S // 2
    wsb = hy.filter_spectrum_workspace(R, 3, [g, g, g], circular)
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(Kern.reshape(R, -1)), H, rows=R, ndim=3, dims=[g, g, g],
                             circular=circular, ws=ws)
    return H


def gpu_nd(u, H, *, circular, gate=None, skip=None, H_batch_stride=0):
    B, D = u.shape[:2]
    dims = list(u.shape[2:])
    ws = torch.empty(max(hy.nd_conv_workspace(dims, B, D, circular), 1), dtype=torch.uint8, device="cuda")
    y = torch.empty_like(u)
    hy.hyena_nd_conv(u, H, y, H_batch_stride=H_batch_stride, circular=circular, Dskip=skip, gate=gate, ws=ws)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("g,circular,per_sample,skip,gate", [
    (4, False, False, True, True),
    (8, False, True, True, True),
    (8, True, False, False, True),
    (16, True, True, True, False),
])
def test_nd_small_grids_direct(g, circular, per_sample, skip, gate):
    rng = np.random.default_rng(g * 10 + circular)
    B, D = 2, 3
    S = g if circular else 2 * g
    nk = B * D if per_sample else D
    Kern = rng.standard_normal((nk, S, S, S)).astype(np.float32)
    if not circular:   # offset -g is outside the non-circular support
        Kern[:, S // 2] = 0
        Kern[:, :, S // 2] = 0
        Kern[:, :, :, S // 2] = 0
    v = rng.standard_normal((B, D, g, g, g)).astype(np.float32)
    x1 = rng.standard_normal((B, D, g, g, g)).astype(np.float32)
    Dk = rng.standard_normal(D).astype(np.float32)
    H = gpu_spectrum3(Kern, circular)
    Href = np.fft.rfftn(Kern.astype(np.float64), axes=(1, 2, 3))
    Hg = H.cpu().numpy().astype(np.complex128)
    check(np.stack([Hg.real, Hg.imag]), np.stack([Href.real, Href.imag]), "f32", "3-D spectrum")
    stride = D * S * S * (S // 2 + 1) if per_sample else 0
    y = gpu_nd(f32_dev(v), H, circular=circular, gate=f32_dev(x1) if gate else None,
               skip=f32_dev(Dk) if skip else None, H_batch_stride=stride)
    got = to_np(y)
    pts = np.arange(g ** 3)
    for b in range(B):
        for d in range(D):
            kern = Kern[b * D + d] if per_sample else Kern[d]
            ref = oracle.nd_conv_points(kern, v[b, d], x1[b, d] if gate else None,
                                        float(Dk[d]) if skip else 0.0, pts, circular).reshape(g, g, g)
            check(got[b, d], ref, "f32", "N-D g%d b%d d%d" % (g, b, d))


def test_nd_delta_and_shift_kernels():
    g, S = 8, 16
    K = np.zeros((2, S, S, S), np.float32)
    K[0, 0, 0, 0] = 1.0                      # identity
    K[1, 1, 2, S - 3] = 1.0                  # shift by (+1, +2, -3)
    H = gpu_spectrum3(K)
    v = np.random.default_rng(1).standard_normal((1, 2, g, g, g)).astype(np.float32)
    got = to_np(gpu_nd(f32_dev(v), H, circular=False))
    np.testing.assert_allclose(got[0, 0], v[0, 0], atol=1e-5)
    sh = np.zeros((g, g, g), np.float32)
    sh[1:, 2:, :g - 3] = v[0, 1, :g - 1, :g - 2, 3:]
    np.testing.assert_allclose(got[0, 1], sh, atol=1e-5)


def test_nd_two_chunk_pipelines_match_one():
    """64^3 slabs on the 128^3 transform grid, more slabs than one ~80 MB
    chunk holds (9 spectra, 19 convolution slabs per chunk): with the
    recommended workspace (two chunk buffers) consecutive chunks alternate
    between the caller's stream and the library's second stream; with the
    minimum (one buffer) they run on the caller's stream alone.  Spectra and
    gated convolutions of the two runs are equal bit for bit, and sampled
    slabs of different chunks match the FFT-route oracle."""
    g, D = 64, 40
    S = 2 * g
    rng = np.random.default_rng(6440)
    K = rng.standard_normal((D, S, S, S)).astype(np.float32)
    K *= np.exp(-np.abs(np.fft.fftfreq(S) * S)[None, :, None, None] / 8).astype(np.float32)
    hd = f32_dev(K.reshape(D, -1))
    per_s = S * S * (S // 2 + 1) * 8
    full = hy.filter_spectrum_workspace(D, 3, [g, g, g])
    assert full == 2 * 9 * per_s
    Hs = []
    for wsb in (full, 9 * per_s):
        H = torch.empty((D, S, S, S // 2 + 1), dtype=torch.complex64, device="cuda")
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        hy.hyena_filter_spectrum(hd, H, rows=D, ndim=3, dims=[g, g, g], ws=ws)
        torch.cuda.current_stream().synchronize()
        Hs.append(H)
    assert torch.equal(torch.view_as_real(Hs[0]), torch.view_as_real(Hs[1]))
    H = Hs[0]
    del Hs
    v = rng.standard_normal((1, D, g, g, g)).astype(np.float32)
    x1 = rng.standard_normal((1, D, g, g, g)).astype(np.float32)
    vd, xd = f32_dev(v), f32_dev(x1)
    per_c = g * S * (S // 2 + 1) * 8
    wfull = hy.nd_conv_workspace([g, g, g], 1, D)
    assert wfull == 2 * 19 * per_c
    ys = []
    for wsb in (wfull, 19 * per_c):
        y = torch.empty_like(vd)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        hy.hyena_nd_conv(vd, H, y, gate=xd, ws=ws)
        torch.cuda.current_stream().synchronize()
        ys.append(y)
    assert torch.equal(ys[0], ys[1])
    got = to_np(ys[0])
    for d in (0, 18, 19, 39):
        ref = oracle.fft_nd_conv(K[d], v[0, d], x1[0, d], 0.0, False)
        check(got[0, d], ref, "f32", "two-lane N-D conv slab %d" % d)


def test_nd_filter_gen_3d_vs_oracle():
    g, F = 8, 4
    w = hw.make("c4", seed=44, B=2, D=6, grid=(g, g, g), with_signals=False)
    S = 2 * g
    h = torch.empty((2, 6, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=F, film_gamma=f32_dev(w.film_gamma),
                        film_beta=f32_dev(w.film_beta), n_sets=2)
    torch.cuda.synchronize()
    got = to_np(h)
    idx = np.arange(S ** 3)
    for b in range(2):
        ref = oracle.filter_gen_3d_points(g, False, F, w.Ws, w.bs, w.film_gamma[b], w.film_beta[b], w.alpha, idx)
        check(got[b].reshape(6, -1), ref.T, "f32", "3-D filters sample %d" % b)


@pytest.mark.parametrize("g,circular,hidden,nout", [(2, True, [16], 5), (2, False, [24, 12], 3), (4, True, [64], 130)])
def test_nd_filter_gen_small_grids(g, circular, hidden, nout):
    """Grids smaller than one 64-position tile, several hidden layers and a
    last layer wider than one 128-output tile, with FiLM on two sets."""
    F = 3
    rng = np.random.default_rng(g * 100 + nout)
    widths = [6 * F] + hidden + [nout]
    Ws, bs = [], []
    for a, b in zip(widths[:-1], widths[1:]):
        Ws.append(rng.uniform(-1 / np.sqrt(a), 1 / np.sqrt(a), (b, a)).astype(np.float32))
        bs.append(rng.uniform(-1 / np.sqrt(a), 1 / np.sqrt(a), b).astype(np.float32))
    alpha = rng.uniform(0.5, 3.0, nout).astype(np.float32)
    gam = rng.normal(0, 0.1, (2, hidden[0])).astype(np.float32)
    bet = rng.normal(0, 0.1, (2, hidden[0])).astype(np.float32)
    S = g if circular else 2 * g
    h = torch.empty((2, nout, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, circular=circular, Ws=[f32_dev(a) for a in Ws],
                        bs=[f32_dev(a) for a in bs], alpha=f32_dev(alpha), n_freq=F,
                        film_gamma=f32_dev(gam), film_beta=f32_dev(bet), n_sets=2)
    torch.cuda.synchronize()
    got = to_np(h)
    idx = np.arange(S ** 3)
    for b in range(2):
        ref = oracle.filter_gen_3d_points(g, circular, F, Ws, bs, gam[b], bet[b], alpha, idx)
        check(got[b].reshape(nout, -1), ref.T, "f32", "3-D filters g%d circ%d set %d" % (g, circular, b))


@pytest.mark.parametrize("engine", ["tensor", "tensor_last", "simt"])
@pytest.mark.parametrize("act,hidden,nout", [("silu", 64, 130), ("sine", 40, 24)])
def test_nd_filter_gen_tensor_core_grid(act, hidden, nout, engine, monkeypatch):
    """A grid with enough 128-position tiles for the tensor-core filter
    kernels (g = 16: 32^3 positions per set, two FiLM sets): both layers on
    the tensor cores (the default for one hidden layer of <= 64 units: the
    3-D encoding of each position written into the first MMA operand), the
    last layer alone, and the FP32 pipes; 130 outputs take two output slices
    (128 + 2), the SIREN case the Gaussian window.  Every voxel and output
    against the oracle."""
    monkeypatch.setenv("HYENA_FILTER_ENGINE", engine)
    g, F = 16, 3
    rng = np.random.default_rng(1600 + nout)
    widths = [6 * F, hidden, nout]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.5, 3.0, nout).astype(np.float32)
    gam = rng.normal(0, 0.1, (2, hidden)).astype(np.float32)
    bet = rng.normal(0, 0.1, (2, hidden)).astype(np.float32)
    sine = act == "sine"
    omega = rng.uniform(1, 4, hidden).astype(np.float32) if sine else None
    S = 2 * g
    h = torch.empty((2, nout, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, film_gamma=f32_dev(gam), film_beta=f32_dev(bet), n_sets=2,
                        act=hy.HY_ACT_SINE if sine else hy.HY_ACT_SILU,
                        omega=f32_dev(omega) if sine else None, window=hy.HY_WIN_GAUSS if sine else hy.HY_WIN_EXP)
    torch.cuda.synchronize()
    got = to_np(h)
    idx = np.arange(S ** 3)
    for b in range(2):
        kw = dict(act="sine", omega=omega, window="gauss") if sine else {}
        ref = oracle.filter_gen_3d_points(g, False, F, Ws, bs, gam[b], bet[b], alpha, idx, **kw)
        check(got[b].reshape(nout, -1), ref.T, "f32", "3-D filters g16 %s %s set %d" % (act, engine, b))


def test_nd_filter_gen_three_layers_few_tiles():
    """3-D filters with two hidden layers and 300 outputs on a small grid
    (g = 8: 16^3 positions = 32 tiles per set, two FiLM sets): all three
    layers on the tensor cores with grid z = 2 over the 3 output slices (the
    last one 44 wide); every voxel and output against the oracle."""
    g, F, nout = 8, 3, 300
    rng = np.random.default_rng(8300)
    widths = [6 * F, 64, 32, nout]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.5, 3.0, nout).astype(np.float32)
    gam = rng.normal(0, 0.1, (2, 64)).astype(np.float32)
    bet = rng.normal(0, 0.1, (2, 64)).astype(np.float32)
    S = 2 * g
    h = torch.empty((2, nout, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, film_gamma=f32_dev(gam), film_beta=f32_dev(bet), n_sets=2)
    torch.cuda.synchronize()
    got = to_np(h)
    idx = np.arange(S ** 3)
    for b in range(2):
        ref = oracle.filter_gen_3d_points(g, False, F, Ws, bs, gam[b], bet[b], alpha, idx)
        check(got[b].reshape(nout, -1), ref.T, "f32", "three-layer 3-D filters set %d" % b)


@pytest.mark.parametrize("circular", [False, True])
def test_nd_filter_gen_siren_gaussian(circular):
    """HyenaND kernel synthesis: SIREN hidden layers (sin of per-unit
    frequencies, FiLM on the first) under the Gaussian window."""
    g, F, nout = 8, 3, 20
    rng = np.random.default_rng(31 + circular)
    widths = [6 * F, 32, 24, nout]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    # frequencies kept where fp32 pre-activations still give ~1e-6 phase error (the
    # map x -> sin(omega x) amplifies rounding by omega)
    omega = np.concatenate([rng.uniform(1, 8, 32), rng.uniform(0.5, 2, 24)]).astype(np.float32)
    alpha = rng.uniform(0.5, 4.0, nout).astype(np.float32)
    gam = rng.normal(0, 0.1, (2, 32)).astype(np.float32)
    bet = rng.normal(0, 0.1, (2, 32)).astype(np.float32)
    S = g if circular else 2 * g
    h = torch.empty((2, nout, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, circular=circular, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, film_gamma=f32_dev(gam), film_beta=f32_dev(bet), n_sets=2,
                        act=hy.HY_ACT_SINE, omega=f32_dev(omega), window=hy.HY_WIN_GAUSS)
    torch.cuda.synchronize()
    got = to_np(h)
    idx = np.arange(S ** 3)
    for b in range(2):
        ref = oracle.filter_gen_3d_points(g, circular, F, Ws, bs, gam[b], bet[b], alpha, idx, act="sine",
                                          omega=omega, window="gauss")
        check(got[b].reshape(nout, -1), ref.T, "f32", "SIREN/Gaussian 3-D filters circ%d set %d" % (circular, b))


def test_c4_full_size():
    """Workload 4 at full size: per-sample FiLM filters on the 128^3 transform
    grid, their spectra and the gated convolution of B2 D128 64^3.  Four slabs
    are checked on all voxels against the FFT-route reference and on 2048
    voxels (plus the 8 corners) against the direct definition."""
    w = hw.make("c4")
    s = w.spec
    B, D, g = s["B"], s["D"], s["grid"][0]
    S = 2 * g
    dev = "cuda"
    h = torch.empty((B, D, S, S, S), device=dev)
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=s["F"], film_gamma=f32_dev(w.film_gamma),
                        film_beta=f32_dev(w.film_beta), n_sets=B)
    H = torch.empty((B, D, S, S, S // 2 + 1), dtype=torch.complex64, device=dev)
    ws = torch.empty(hy.filter_spectrum_workspace(B * D, 3, [g, g, g]), dtype=torch.uint8, device=dev)
    hy.hyena_filter_spectrum(h, H, rows=B * D, ndim=3, dims=[g, g, g], ws=ws)
    del ws
    u = f32_dev(w.v.f32)
    x1 = f32_dev(w.xs[0].f32)
    y = gpu_nd(u, H, circular=False, gate=x1, H_batch_stride=D * S * S * (S // 2 + 1))
    got = to_np(y)
    assert np.all(np.isfinite(got))
    slabs = [(0, 0), (0, 77), (1, 3), (1, 127)]
    rng = np.random.default_rng(4)
    pts = np.concatenate([rng.choice(g ** 3, 2048, replace=False),
                          [0, g - 1, g * (g - 1), g * g - 1, g ** 3 - g * g, g ** 3 - g * (g - 1) - 1,
                           g ** 3 - g, g ** 3 - 1]])
    idx = np.arange(S ** 3)
    for b, d in slabs:
        Ws = list(w.Ws[:-1]) + [w.Ws[-1][[d]]]
        bs = list(w.bs[:-1]) + [w.bs[-1][[d]]]
        kern = oracle.filter_gen_3d_points(g, False, s["F"], Ws, bs, w.film_gamma[b], w.film_beta[b],
                                           w.alpha[[d]], idx)[:, 0].reshape(S, S, S)
        check(to_np(h[b, d]), kern, "f32", "c4 filter b%d d%d" % (b, d))
        ref = oracle.fft_nd_conv(kern, w.v.f32[b, d], w.xs[0].f32[b, d])
        check(got[b, d], ref, "f32", "c4 slab b%d d%d (FFT route)" % (b, d))
        direct = oracle.nd_conv_points(kern, w.v.f32[b, d], w.xs[0].f32[b, d], 0.0, pts)
        check_part(got[b, d].ravel()[pts], direct, float(np.sqrt(np.mean(ref ** 2))), "f32",
                   "c4 slab b%d d%d voxels (direct)" % (b, d))


def test_nd_filter_gen_resident_weights_film():
    """3-D kernels on a 64^3 transform grid (g = 32), FiLM on two sets: the
    persistent resident-weight filter kernel; sampled grid points of both
    sets against the oracle (with the support mask)."""
    g, F, nout = 32, 4, 12
    rng = np.random.default_rng(3232)
    widths = [6 * F, 32, nout]
    Ws = [rng.uniform(-1, 1, (b, a)).astype(np.float32) / np.sqrt(a) for a, b in zip(widths[:-1], widths[1:])]
    bs = [rng.uniform(-0.5, 0.5, b).astype(np.float32) for b in widths[1:]]
    alpha = rng.uniform(0.5, 3.0, nout).astype(np.float32)
    gam = rng.normal(0, 0.1, (2, 32)).astype(np.float32)
    bet = rng.normal(0, 0.1, (2, 32)).astype(np.float32)
    S = 2 * g
    h = torch.empty((2, nout, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in Ws], bs=[f32_dev(a) for a in bs],
                        alpha=f32_dev(alpha), n_freq=F, film_gamma=f32_dev(gam), film_beta=f32_dev(bet), n_sets=2)
    torch.cuda.synchronize()
    got = to_np(h).reshape(2, nout, -1)
    idx = np.random.default_rng(5).choice(S ** 3, 20000, replace=False)
    for b in range(2):
        ref = oracle.filter_gen_3d_points(g, False, F, Ws, bs, gam[b], bet[b], alpha, idx)
        check(got[b][:, idx], ref.T, "f32", "resident-weight 3-D filters set %d" % b)
