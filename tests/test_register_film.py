"""HyenaND input conditioning ([ND] 레지스터 및 FiLM): the softmax-weighted
mean of register activations, z(x), and the FiLM parameters it drives,
against the float64 oracle; then the whole conditioned path -- registers ->
(gamma, beta) -> 3-D kernel synthesis -> kernel spectra -> gated N-D
convolution -- on a small grid against the oracle's direct N-D sum."""
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


@pytest.mark.parametrize("B,R,C,H,use_q,use_s,use_b", [
    (2, 4, 64, 64, True, False, True),
    (3, 1, 5, 3, False, True, False),
    (1, 7, 33, 9, False, False, True),
    (4, 37, 300, 40, True, True, True),
    (2, 1024, 8192, 2, True, True, False),
])
def test_register_film_vs_oracle(B, R, C, H, use_q, use_s, use_b):
    rng = np.random.default_rng(B * 1000 + R + C)
    reg = rng.standard_normal((B, R, C)).astype(np.float32)
    q = (rng.standard_normal(C) / np.sqrt(C)).astype(np.float32) if use_q else None
    sc = (3 * rng.standard_normal((B, R))).astype(np.float32) if use_s else None
    W = (rng.standard_normal((2 * H, C)) / np.sqrt(C)).astype(np.float32)
    bb = rng.standard_normal(2 * H).astype(np.float32) if use_b else None
    gam = torch.empty((B, H), device="cuda")
    bet = torch.empty((B, H), device="cuda")
    hy.hyena_register_film(f32_dev(reg), f32_dev(W), gam, bet, query=f32_dev(q) if use_q else None,
                           scores=f32_dev(sc) if use_s else None, b_film=f32_dev(bb) if use_b else None)
    torch.cuda.synchronize()
    g_ref, b_ref, _, _ = oracle.register_film(reg, q, sc, W, bb if use_b else np.zeros(2 * H))
    check(to_np(gam), g_ref, "f32", "register FiLM gamma B%d R%d C%d" % (B, R, C))
    check(to_np(bet), b_ref, "f32", "register FiLM beta B%d R%d C%d" % (B, R, C))


def test_register_conditioned_nd_path_end_to_end():
    """z(x) -> FiLM -> 3-D kernels -> spectra -> gated N-D convolution,
    both samples, every voxel of a small grid against the direct sum."""
    g = 8
    w = hw.make("c4", seed=4400, B=2, D=3, grid=(g, g, g), registers=6, register_width=48)
    s = w.spec
    B, D, S = 2, 3, 2 * g
    H = s["hidden"][0]
    gam = torch.empty((B, H), device="cuda")
    bet = torch.empty((B, H), device="cuda")
    hy.hyena_register_film(f32_dev(w.reg), f32_dev(w.film_W), gam, bet, query=f32_dev(w.reg_query),
                           b_film=f32_dev(w.film_b))
    h = torch.empty((B, D, S, S, S), device="cuda")
    hy.hyena_filter_gen(h, ndim=3, grid=g, Ws=[f32_dev(a) for a in w.Ws], bs=[f32_dev(a) for a in w.bs],
                        alpha=f32_dev(w.alpha), n_freq=s["F"], film_gamma=gam, film_beta=bet, n_sets=B)
    Hs = torch.empty((B, D, S, S, S // 2 + 1), dtype=torch.complex64, device="cuda")
    ws = torch.empty(max(hy.filter_spectrum_workspace(B * D, 3, [g, g, g]),
                         hy.nd_conv_workspace([g, g, g], B, D), 1), dtype=torch.uint8, device="cuda")
    hy.hyena_filter_spectrum(h, Hs, rows=B * D, ndim=3, dims=[g, g, g], ws=ws)
    u, x1 = f32_dev(w.v.f32), f32_dev(w.xs[0].f32)
    y = torch.empty_like(u)
    hy.hyena_nd_conv(u, Hs, y, H_batch_stride=D * S * S * (S // 2 + 1), gate=x1, ws=ws)
    torch.cuda.synchronize()
    g_ref, b_ref, _, _ = oracle.register_film(w.reg, w.reg_query, None, w.film_W, w.film_b)
    check(to_np(gam), g_ref, "f32", "registers -> gamma")
    pts = np.arange(g ** 3)
    for b in range(B):
        K = oracle.filter_gen_3d(g, False, s["F"], w.Ws, w.bs, g_ref[b], b_ref[b], w.alpha)
        for d in range(D):
            ref = oracle.nd_conv_points(K[d], w.v.f32[b, d], w.xs[0].f32[b, d], 0.0, pts, False)
            check(to_np(y[b, d]).ravel(), ref, "f32", "register-conditioned N-D conv b%d d%d" % (b, d))
