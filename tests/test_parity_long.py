"""Parity of the multi-pass (four-step) path for sequences longer than one CTA
can hold (L > 16384) against the float64 oracle: the gated chain at several
lengths (ragged and power-of-two), orders 2 and 3, fp32 and bf16 I/O, the long
filter spectrum, and workload 3 at full size (B1 D256 L=2^20, order 3)."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import check, check_part, f32_dev, to_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _filters(rng, K, D, L):
    t = np.arange(L)
    rate = rng.uniform(0.1, 2.0, size=(K, D, 1))
    return (rng.standard_normal((K, D, L)) * np.exp(-rate * t / L)).astype(np.float32)


def _spectra(h32):
    K, D, L = h32.shape
    nb = hy.spectrum_bins(L)
    hd = f32_dev(h32.reshape(K * D, L))
    H = torch.empty((K * D, nb), dtype=torch.complex64, device="cuda")
    wsb = hy.filter_spectrum_workspace(K * D, 1, [L])
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    hy.hyena_filter_spectrum(hd, H, rows=K * D, ndim=1, dims=[L], ws=ws)
    return [H[k * D:(k + 1) * D] for k in range(K)], H


def _run(v, xs, Hs, dsk, L, B, D, order, code):
    y = torch.empty_like(v)
    wsb = hy.operator_workspace(order, B, D, L, code)
    assert wsb > 0
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    hy.hyena_operator(v, xs, Hs, y, Dskips=dsk, ws=ws)
    torch.cuda.synchronize()
    return y


def test_two_chunk_pipelines_match_one():
    """More rows than one ~104 MB chunk holds (L = 2^15: 416 rows per chunk;
    1000 rows = 3 chunks, the last one ragged): with the recommended
    workspace (two chunk buffers) consecutive chunks alternate between the
    caller's stream and the library's second stream; with the minimum (one
    chunk buffer) they all run on the caller's stream.  The spectra and the
    order-3 operator outputs of the two runs are equal bit for bit, sampled
    rows of each chunk match the float64 oracle, and the outputs are ordered
    on the caller's stream (read right after its synchronisation)."""
    B, D, L, order = 2, 500, 1 << 15, 3
    K = order - 1
    rows = B * D
    rng = np.random.default_rng(2015)
    h32 = _filters(rng, K, D, L)
    nb = hy.spectrum_bins(L)
    hd = f32_dev(h32.reshape(K * D, L))
    full = hy.filter_spectrum_workspace(K * D, 1, [L])
    one = (416 * 8) << 15
    assert full == 2 * one
    Hs_ = []
    for wsb in (full, one):
        H = torch.empty((K * D, nb), dtype=torch.complex64, device="cuda")
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        hy.hyena_filter_spectrum(hd, H, rows=K * D, ndim=1, dims=[L], ws=ws)
        torch.cuda.current_stream().synchronize()
        Hs_.append(H)
    assert torch.equal(torch.view_as_real(Hs_[0]), torch.view_as_real(Hs_[1]))
    H = Hs_[0]
    Hs = [H[k * D:(k + 1) * D] for k in range(K)]
    v = torch.randn(B, D, L, device="cuda")
    xs = [torch.randn(B, D, L, device="cuda") for _ in range(K)]
    dsk = [f32_dev(rng.standard_normal(D).astype(np.float32)) for _ in range(K)]
    wfull = hy.operator_workspace(order, B, D, L, 0)
    assert wfull == 2 * one
    ys = []
    for wsb in (wfull, one):
        y = torch.empty_like(v)
        ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
        hy.hyena_operator(v, xs, Hs, y, Dskips=dsk, ws=ws)
        torch.cuda.current_stream().synchronize()
        ys.append(y)
    assert torch.equal(ys[0], ys[1])
    pick = np.array([0, 415, 416, 500, 831, 832, 999])      # rows of each chunk, both lanes
    Dsk = np.stack([to_np(dk) for dk in dsk])
    ref = oracle.fft_hyena_rows(to_np(v), [to_np(x) for x in xs], h32.astype(np.float64), Dsk, rows=pick)
    check(to_np(ys[0]).reshape(rows, L)[pick], ref, "f32", "two-lane operator sampled rows")


def test_two_chunk_pipelines_in_a_cuda_graph():
    """The multi-pass operator with two chunk pipelines (L = 2^15, 1000 rows:
    three chunks) captured into a CUDA graph on a side stream: the second
    stream forks off the captured stream and joins it by events, so the
    capture holds both chunk sequences; two replays give the eager result
    bit for bit."""
    B, D, L, order = 2, 500, 1 << 15, 2
    rng = np.random.default_rng(3215)
    h32 = _filters(rng, 1, D, L)
    Hs, _ = _spectra(h32)
    v = torch.randn(B, D, L, device="cuda")
    xs = [torch.randn(B, D, L, device="cuda")]
    wsb = hy.operator_workspace(order, B, D, L, 0)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    y_eager = torch.empty_like(v)
    hy.hyena_operator(v, xs, Hs, y_eager, ws=ws)
    torch.cuda.synchronize()
    y = torch.zeros_like(v)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        hy.hyena_operator(v, xs, Hs, y, ws=ws)          # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    y.zero_()
    with torch.cuda.graph(g):
        hy.hyena_operator(v, xs, Hs, y, ws=ws)
    for _ in range(2):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y, y_eager)
    del g


LONG = [
    # B, D, L, order, dtype, skip
    (1, 2, 20000, 2, "f32", True),
    (2, 1, 32768, 3, "f32", True),
    (1, 3, 40000, 2, "bf16", True),
    (1, 2, 65536, 2, "f32", False),
    (1, 1, 30001, 2, "f32", True),      # odd length: scalar tails of the vector loads
    (1, 1, 50002, 3, "bf16", True),     # L = 2 (mod 4)
]


@pytest.mark.parametrize("B,D,L,order,dtype,skip", LONG)
def test_long_operator_vs_direct(B, D, L, order, dtype, skip):
    w = hw.make("c3", seed=3000 + L, B=B, D=D, L=L, order=order, dtype=dtype, skip=skip)
    rng = np.random.default_rng(L)
    K = order - 1
    h32 = _filters(rng, K, D, L)
    Hs, H = _spectra(h32)
    Href = oracle.fft_spectrum(h32.reshape(K * D, L), n=2 * (hy.spectrum_bins(L) - 1))
    Hg = H.cpu().numpy().astype(np.complex128)
    check(np.stack([Hg.real, Hg.imag]), np.stack([Href.real, Href.imag]), "f32", "long spectrum")
    v = to_dev(w.v, dtype)
    xs = [to_dev(x, dtype) for x in w.xs]
    dsk = [f32_dev(w.Dskip[k]) for k in range(K)] if skip else None
    y = _run(v, xs, Hs, dsk, L, B, D, order, 1 if dtype == "bf16" else 0)
    ref = oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], h32.astype(np.float64),
                            w.Dskip if skip else None)
    check(to_np(y).reshape(B * D, L), ref, dtype, "long operator L%d order%d" % (L, order))


def test_long_operator_misaligned_rows_bitwise():
    """Signals that are 8- but not 16-byte aligned take the scalar load/store
    path of the column passes; it must give bit-identical results to the
    vector path on the same values."""
    B, D, L, order = 1, 2, 36000, 3
    w = hw.make("c3", seed=5, B=B, D=D, L=L, order=order)
    h32 = _filters(np.random.default_rng(5), 2, D, L)
    Hs, _ = _spectra(h32)
    dsk = [f32_dev(w.Dskip[k]) for k in range(2)]

    # 8 bytes past a 256-byte boundary: allowed (rows of even length need
    # 8-byte alignment) but not 16-byte aligned
    def shifted(a):
        flat = torch.zeros(a.size + 2, device="cuda")
        flat[2:] = torch.from_numpy(np.ascontiguousarray(a, np.float32).ravel()).cuda()
        return flat[2:].view(a.shape)

    y0 = _run(f32_dev(w.v.f32), [f32_dev(x.f32) for x in w.xs], Hs, dsk, L, B, D, order, 0)
    v1 = shifted(w.v.f32)
    xs1 = [shifted(x.f32) for x in w.xs]
    y1 = torch.empty(B * D * L + 2, device="cuda")[2:].view(B, D, L)
    wsb = hy.operator_workspace(order, B, D, L, 0)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda")
    hy.hyena_operator(v1, xs1, Hs, y1, Dskips=dsk, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)


def test_long_operator_2p18_fft_reference():
    B, D, L, order = 1, 2, 1 << 18, 3
    w = hw.make("c3", seed=77, B=B, D=D, L=L)
    h32 = _filters(np.random.default_rng(9), 2, D, L)
    Hs, _ = _spectra(h32)
    v = to_dev(w.v, "f32")
    xs = [to_dev(x, "f32") for x in w.xs]
    y = _run(v, xs, Hs, [f32_dev(w.Dskip[k]) for k in range(2)], L, B, D, order, 0)
    got = to_np(y).reshape(B * D, L)
    ref = oracle.fft_hyena_rows(w.v.f32, [x.f32 for x in w.xs], h32.astype(np.float64), w.Dskip)
    check(got, ref, "f32", "L=2^18 vs FFT route")
    pre = oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], h32.astype(np.float64), w.Dskip, T=2048)
    for r in range(B * D):
        rms = float(np.sqrt(np.mean(ref[r] ** 2)))
        check_part(got[r, :2048], pre[r], rms, "f32", "L=2^18 prefix vs direct")


def test_c3_full_size():
    """Workload 3 at full size: implicit filters 17->64->(2*256) on L = 2^20,
    their spectra and the order-3 operator in fp32.  Eight rows are checked
    against the FFT-route reference (all samples), their first 2048 samples
    against the direct chain, and late samples of the last order directly."""
    w = hw.make("c3")
    s = w.spec
    B, D, L, K = s["B"], s["D"], s["L"], 2
    dev = "cuda"
    h = torch.empty((K * D, L), device=dev)
    hy.hyena_filter_gen(h, ndim=1, L=L, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=s["F"], include_t=True)
    nb = hy.spectrum_bins(L)
    H = torch.empty((K * D, nb), dtype=torch.complex64, device=dev)
    ws = torch.empty(hy.filter_spectrum_workspace(K * D, 1, [L]), dtype=torch.uint8, device=dev)
    hy.hyena_filter_spectrum(h, H, rows=K * D, ndim=1, dims=[L], ws=ws)
    del ws
    v = to_dev(w.v, "f32")
    xs = [to_dev(x, "f32") for x in w.xs]
    y = _run(v, xs, [H[:D], H[D:]], [f32_dev(w.Dskip[k]) for k in range(K)], L, B, D, 3, 0)
    got = to_np(y).reshape(B * D, L)
    assert np.all(np.isfinite(got))
    chans = np.array([0, 37, 128, 255])
    # oracle filters for those channels only (last layer restricted to their columns)
    cols = np.concatenate([chans, D + chans])
    Ws = list(w.Ws[:-1]) + [w.Ws[-1][cols]]
    bs = list(w.bs[:-1]) + [w.bs[-1][cols]]
    h64 = oracle.filter_gen_1d(L, s["F"], True, Ws, bs, w.alpha[cols])        # (2*4, L)
    hgot = to_np(h[torch.as_tensor(cols, device=dev)])
    check(hgot, h64, "f32", "c3 filters")
    del h
    hk = np.zeros((K, D, L))
    hk[0, chans] = h64[:4]
    hk[1, chans] = h64[4:]
    ref = oracle.fft_hyena_rows(w.v.f32, [x.f32 for x in w.xs], hk, w.Dskip, rows=chans)
    check(got[chans], ref, "f32", "c3 sampled rows vs FFT route")
    pre = oracle.hyena_rows(w.v.f32, [x.f32 for x in w.xs], hk, w.Dskip, rows=chans, T=2048)
    for i, c in enumerate(chans):
        rms = float(np.sqrt(np.mean(ref[i] ** 2)))
        check_part(got[c, :2048], pre[i], rms, "f32", "c3 prefix vs direct chain")
    # late samples of the last order, directly, on top of the float64 first order
    z1 = oracle.fft_hyena_rows(w.v.f32, [w.xs[0].f32], hk[:1], w.Dskip[:1], rows=chans)
    ts = np.array([L // 2 + 3, L - 1000, L - 1])
    for i, c in enumerate(chans):
        d = oracle.conv_gate_samples(hk[1, c], z1[i], w.xs[1].f32[0, c], float(w.Dskip[1, c]), ts)
        check_part(got[c, ts], d, float(np.sqrt(np.mean(ref[i] ** 2))), "f32", "c3 late samples, direct")


def test_long_spectrum_matches_reference():
    L = 1 << 20
    rng = np.random.default_rng(4)
    h32 = _filters(rng, 1, 3, L)
    _, H = _spectra(h32)
    ref = oracle.fft_spectrum(h32.reshape(3, L))
    Hg = H.cpu().numpy().astype(np.complex128)
    check(np.stack([Hg.real, Hg.imag]), np.stack([ref.real, ref.imag]), "f32", "spectrum L=2^20")
    # a delta filter has a unit spectrum; a shifted delta a pure phase ramp
    hd = np.zeros((2, L), np.float32)
    hd[0, 0] = 1
    hd[1, 12345] = 1
    _, Hd = _spectra(hd.reshape(1, 2, L))
    Hd = Hd.cpu().numpy().astype(np.complex128)
    k = np.arange(L + 1)
    np.testing.assert_allclose(Hd[0], np.ones(L + 1), atol=1e-6)
    np.testing.assert_allclose(Hd[1], np.exp(-2j * np.pi * k * 12345 / (2 * L)), atol=2e-6)


def test_long_spectrum_ragged_length():
    """A filter length that is neither a power of two nor a multiple of 4."""
    L = 70001
    h32 = _filters(np.random.default_rng(6), 1, 2, L)
    _, H = _spectra(h32)
    ref = oracle.fft_spectrum(h32.reshape(2, L), n=2 * (hy.spectrum_bins(L) - 1))
    Hg = H.cpu().numpy().astype(np.complex128)
    check(np.stack([Hg.real, Hg.imag]), np.stack([ref.real, ref.imag]), "f32", "spectrum L=70001")
