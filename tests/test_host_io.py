"""Host-buffer entry points: the operator and the spectral gate with their
signals in page-locked host memory, copied in, computed and copied out chunk
by chunk on three streams.  Each chunk runs the device entry point's kernels
on a subset of rows, so the results must equal the device path bit for bit;
the shapes make several chunks, more than the 3 ring slots, on the on-chip
and the multi-pass operator, the N-D convolution and the gate."""
import numpy as np
import pytest

from _helpers import f32_dev

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


def _pinned(t):
    return t.cpu().pin_memory()


def _spectra(rng, rows, L):
    t = np.arange(L)
    h = (rng.standard_normal((rows, L)) * np.exp(-rng.uniform(0.2, 3.0, (rows, 1)) * t / L)).astype(np.float32)
    H = torch.empty((rows, hy.spectrum_bins(L)), dtype=torch.complex64, device="cuda")
    wsb = hy.filter_spectrum_workspace(rows, 1, [L])
    ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(h), H, rows=rows, ndim=1, dims=[L], ws=ws)
    return H


@pytest.mark.parametrize("B,D,L,order,dtype", [
    (2, 768, 8192, 2, torch.float32),    # 2 chunks per batch of 512 channels: 4 chunks
    (5, 600, 8192, 2, torch.bfloat16),   # one whole batch per chunk: 5 chunks
    (1, 300, 40000, 3, torch.float32),   # multi-pass: 3 chunks of <= 104 rows
])
def test_operator_host_matches_device(B, D, L, order, dtype):
    rng = np.random.default_rng(L + D)
    K = order - 1
    H = _spectra(rng, K * D, L)
    Hs = [H[k * D:(k + 1) * D] for k in range(K)]
    dsk = [f32_dev(rng.standard_normal(D).astype(np.float32)) for _ in range(K)]
    v = torch.randn((B, D, L), device="cuda").to(dtype)
    xs = [torch.randn((B, D, L), device="cuda").to(dtype) for _ in range(K)]
    code = hy.HY_BF16 if dtype == torch.bfloat16 else hy.HY_F32
    y_dev = torch.empty_like(v)
    wsd = hy.operator_workspace(order, B, D, L, code)
    hy.hyena_operator(v, xs, Hs, y_dev, Dskips=dsk,
                      ws=torch.empty(wsd, dtype=torch.uint8, device="cuda") if wsd else None)
    vh, xh = _pinned(v), [_pinned(x) for x in xs]
    yh = torch.full(v.shape, float("nan"), dtype=dtype).pin_memory()
    ws = torch.empty(hy.operator_host_workspace(order, B, D, L, code), dtype=torch.uint8, device="cuda")
    hy.hyena_operator_host(vh, xh, Hs, yh, Dskips=dsk, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())
    # a second call on the same ring gives the same result
    yh2 = torch.empty_like(yh).pin_memory()
    hy.hyena_operator_host(vh, xh, Hs, yh2, Dskips=dsk, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh2, yh)


def test_spectral_gate_host_matches_device():
    B, Hh, Dh, L = 3, 10, 64, 32768       # 4 heads per chunk: 3 chunks per batch, 9 chunks
    rng = np.random.default_rng(11)
    M = L // 2
    g = torch.from_numpy((rng.standard_normal((B, Hh, M + 1)) + 1j * rng.standard_normal((B, Hh, M + 1)))
                         .astype(np.complex64)).cuda()
    x = torch.randn((B, Hh, Dh, L), device="cuda").to(torch.bfloat16)
    x2 = torch.randn_like(x)
    y_dev = torch.empty_like(x)
    hy.spectral_gate(x, g, y_dev, x2=x2, g_batch_stride=Hh * (M + 1))
    xh, x2h = _pinned(x), _pinned(x2)
    yh = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    ws = torch.empty(hy.spectral_gate_host_workspace(B, Hh, Dh, L, hy.HY_BF16), dtype=torch.uint8, device="cuda")
    hy.spectral_gate_host(xh, g, yh, x2=x2h, g_batch_stride=Hh * (M + 1), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())


def test_nd_conv_host_matches_device():
    B, D, g = 2, 40, 32                    # 128 KB slabs: 128 per chunk would be whole batches
    S = 2 * g
    rng = np.random.default_rng(12)
    nb = S // 2 + 1
    H = torch.from_numpy((rng.standard_normal((B, D, S, S, nb)) + 1j * rng.standard_normal((B, D, S, S, nb)))
                         .astype(np.complex64) * 1e-3).cuda()
    u = torch.randn((B, D, g, g, g), device="cuda")
    x1 = torch.randn_like(u)
    dsk = f32_dev(rng.standard_normal(D).astype(np.float32))
    stride = D * S * S * nb
    y_dev = torch.empty_like(u)
    wsd = torch.empty(hy.nd_conv_workspace([g, g, g], B, D), dtype=torch.uint8, device="cuda")
    hy.hyena_nd_conv(u, H, y_dev, H_batch_stride=stride, Dskip=dsk, gate=x1, ws=wsd)
    yh = torch.empty(u.shape).pin_memory()
    ws = torch.empty(hy.nd_conv_host_workspace([g, g, g], B, D), dtype=torch.uint8, device="cuda")
    hy.hyena_nd_conv_host(_pinned(u), H, yh, H_batch_stride=stride, Dskip=dsk, gate=_pinned(x1), ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())


def test_nd_conv_host_channel_chunks():
    B, D, g = 2, 24, 64                    # 1 MB slabs: 16 per chunk, 2 chunks per batch
    S = 2 * g
    rng = np.random.default_rng(13)
    nb = S // 2 + 1
    H = torch.from_numpy((rng.standard_normal((D, S, S, nb)) + 1j * rng.standard_normal((D, S, S, nb)))
                         .astype(np.complex64) * 1e-3).cuda()
    u = torch.randn((B, D, g, g, g), device="cuda")
    y_dev = torch.empty_like(u)
    wsd = torch.empty(hy.nd_conv_workspace([g, g, g], B, D), dtype=torch.uint8, device="cuda")
    hy.hyena_nd_conv(u, H, y_dev, ws=wsd)
    yh = torch.empty(u.shape).pin_memory()
    ws = torch.empty(hy.nd_conv_host_workspace([g, g, g], B, D), dtype=torch.uint8, device="cuda")
    hy.hyena_nd_conv_host(_pinned(u), H, yh, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, y_dev.cpu())


def test_host_entry_rejects_device_signals():
    B, D, L = 1, 4, 1024
    v = torch.randn((B, D, L), device="cuda")
    H = _spectra(np.random.default_rng(1), D, L)
    ws = torch.empty(hy.operator_host_workspace(2, B, D, L, hy.HY_F32), dtype=torch.uint8, device="cuda")
    with pytest.raises(hy.HyenaError) as ei:
        hy.hyena_operator_host(v, [v.cpu().pin_memory()], [H], torch.empty((B, D, L)).pin_memory(), ws=ws)
    assert "device memory" in str(ei.value)
