"""Streaming decode of the spectral gate with a prefix-FFT cache, against
the float64 oracle: each step's output equals the full gated circular
convolution of the prefix (later positions zero) at that position; the cache
after T steps equals the DFT of the prefix; a prompt's spectrum from
hyena_filter_spectrum works as the starting cache."""
import numpy as np
import pytest

import hyena_workloads as hw
import oracle
from _helpers import check, f32_dev, to_np

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
import implicit_long_convolution_b200 as hy  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("B,Hh,Dh,n,T,dtype", [
    (2, 3, 4, 64, 64, "f32"),      # every position, cache wraps to the full sequence
    (1, 2, 8, 1024, 200, "f32"),
    (2, 2, 3, 4096, 50, "bf16"),
    (1, 1, 2, 32768, 40, "f32"),   # the largest gate length
])
def test_decode_steps_vs_oracle(B, Hh, Dh, n, T, dtype):
    rng = np.random.default_rng(n + T)
    nb = n // 2 + 1
    g = (rng.standard_normal((B, Hh, nb)) + 1j * rng.standard_normal((B, Hh, nb))).astype(np.complex64)
    x1 = rng.standard_normal((B, Hh, Dh, n)).astype(np.float32)
    x2 = rng.standard_normal((B, Hh, Dh, n)).astype(np.float32)
    if dtype == "bf16":
        x1, x2 = (hw.bf16_to_f32(hw.bf16_round(a)) for a in (x1, x2))
        tdt = torch.bfloat16
    else:
        tdt = torch.float32
    gd = torch.from_numpy(g).cuda()
    cache = torch.zeros((B, Hh, Dh, nb), dtype=torch.complex64, device="cuda")
    xs = torch.from_numpy(x1).cuda().to(tdt)
    x2s = torch.from_numpy(x2).cuda().to(tdt)
    ys = torch.empty((T, B, Hh, Dh), dtype=tdt, device="cuda")
    for pos in range(T):
        hy.spectral_gate_decode(xs[..., pos].contiguous(), gd, cache, ys[pos], pos=pos,
                                x2=x2s[..., pos].contiguous(), g_batch_stride=Hh * nb)
    torch.cuda.synchronize()
    got = to_np(ys)
    ref = np.empty((T, B, Hh, Dh))
    for b in range(B):
        for h in range(Hh):
            for d in range(Dh):
                ref[:, b, h, d] = oracle.prefix_gate_outputs(g[b, h], x1[b, h, d], x2[b, h, d], T)
    check(got, ref, dtype, "decode outputs n=%d" % n)
    pre = x1[..., :T].reshape(-1, T)
    refc = oracle.dft_real_rows(pre, n).reshape(B, Hh, Dh, nb)
    gc = cache.cpu().numpy().astype(np.complex128)
    check(np.stack([gc.real, gc.imag]), np.stack([refc.real, refc.imag]), "f32", "prefix cache n=%d" % n)


def test_decode_from_prompt_spectrum():
    """Prefill: the spectrum of a zero-padded prompt (circular filter
    spectrum) is the cache after the prompt's tokens; decoding continues."""
    B, Hh, Dh, n, P, T = 1, 2, 4, 512, 300, 20
    rng = np.random.default_rng(5)
    nb = n // 2 + 1
    g = (rng.standard_normal((Hh, nb)) + 1j * rng.standard_normal((Hh, nb))).astype(np.complex64)
    x1 = rng.standard_normal((B, Hh, Dh, n)).astype(np.float32)
    prompt = x1.copy()
    prompt[..., P:] = 0
    cache = torch.empty((B, Hh, Dh, nb), dtype=torch.complex64, device="cuda")
    hy.hyena_filter_spectrum(f32_dev(prompt.reshape(-1, n)), cache.view(-1, nb), rows=B * Hh * Dh, ndim=1,
                             dims=[n], circular=True)
    gd = torch.from_numpy(g).cuda()
    xs = torch.from_numpy(x1).cuda()
    ys = torch.empty((T, B, Hh, Dh), device="cuda")
    for i in range(T):
        hy.spectral_gate_decode(xs[..., P + i].contiguous(), gd, cache, ys[i], pos=P + i)
    torch.cuda.synchronize()
    ref = np.empty((T, B, Hh, Dh))
    for h in range(Hh):
        for d in range(Dh):
            ref[:, 0, h, d] = oracle.prefix_gate_outputs(g[h], x1[0, h, d], None, P + T)[P:]
    check(to_np(ys), ref, "f32", "decode after prefill")
