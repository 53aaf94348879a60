"""Pins for the float64 oracle: each check ties an oracle function to something
other than itself -- a closed form, an invariant, a hand-derived fixture, an
independent brute force or a library routine -- so that a dropped term, a wrong
sign or index or a transposed operand fails here.  CPU only."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- a1 PE

def test_pe1d_closed_forms():
    L, F = 64, 8
    pe = oracle.pe1d(L, F, True)
    assert pe.shape == (L, 1 + 2 * F)
    # t = 0: [0, cos 0 = 1 (F times), sin 0 = 0 (F times)]
    np.testing.assert_array_equal(pe[0], np.r_[0.0, np.ones(F), np.zeros(F)])
    # t = L/4: angle pi*j/2 -> cos: 0,-1,0,1,...; sin: 1,0,-1,0,...
    j = np.arange(1, F + 1)
    cos_q = np.array([[1, 0, -1, 0][k % 4] for k in j], float)
    sin_q = np.array([[0, 1, 0, -1][k % 4] for k in j], float)
    np.testing.assert_allclose(pe[L // 4], np.r_[0.25, cos_q, sin_q], atol=1e-15)
    # all t against numpy's cos/sin of the unreduced angle
    t = np.arange(L)[:, None]
    ang = 2 * np.pi * j[None, :] * t / L
    np.testing.assert_allclose(pe[:, 1:1 + F], np.cos(ang), atol=1e-13)
    np.testing.assert_allclose(pe[:, 1 + F:], np.sin(ang), atol=1e-13)
    np.testing.assert_array_equal(pe[:, 0], np.arange(L) / L)
    assert oracle.pe1d(L, F, False).shape == (L, 2 * F)


# ---------------------------------------------------------------- a2 filter MLP

def _np_mlp(x, Ws, bs, gamma=None, beta=None):
    a = x
    for l, (W, b) in enumerate(zip(Ws, bs)):
        a = a @ np.asarray(W, np.float64).T + np.asarray(b, np.float64)
        if l < len(Ws) - 1:
            if l == 0 and gamma is not None:
                a = (1.0 + gamma) * a + beta
            a = a / (1.0 + np.exp(-a))
    return a


def test_filter_gen_constant_output():
    L, F, nout = 32, 4, 5
    rng = np.random.default_rng(0)
    Ws = [rng.standard_normal((16, 9)), np.zeros((nout, 16))]
    c = rng.standard_normal(nout)
    bs = [rng.standard_normal(16), c]
    h0 = oracle.filter_gen_1d(L, F, True, Ws, bs, np.zeros(nout))
    np.testing.assert_array_equal(h0, np.repeat(c[:, None], L, axis=1))
    alpha = np.array([0.0, 0.5, 1.0, 2.0, 3.0])
    h = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha)
    expect = c[:, None] * np.exp(-alpha[:, None] * np.arange(L)[None, :] / L)
    np.testing.assert_allclose(h, expect, rtol=1e-15, atol=0)


@pytest.mark.parametrize("hidden", [[32], [64, 64]])
def test_filter_gen_vs_numpy_mlp(hidden):
    L, F, nout = 128, 8, 24
    rng = np.random.default_rng(1)
    widths = [1 + 2 * F] + hidden + [nout]
    Ws = [rng.uniform(-.5, .5, (widths[i + 1], widths[i])) for i in range(len(widths) - 1)]
    bs = [rng.uniform(-.5, .5, widths[i + 1]) for i in range(len(widths) - 1)]
    alpha = rng.uniform(0.3, 5, nout)
    h = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha)
    t = np.arange(L)
    j = np.arange(1, F + 1)
    pe = np.concatenate([(t / L)[:, None], np.cos(2 * np.pi * np.outer(t, j) / L),
                         np.sin(2 * np.pi * np.outer(t, j) / L)], axis=1)
    ref = _np_mlp(pe, Ws, bs) * np.exp(-np.outer(t, alpha) / L)
    np.testing.assert_allclose(h, ref.T, rtol=1e-12, atol=1e-13)


def test_filter_gen_3d_points():
    g, F, nout = 4, 4, 6
    S = 2 * g
    rng = np.random.default_rng(2)
    widths = [6 * F, 16, nout]
    Ws = [rng.uniform(-.5, .5, (widths[i + 1], widths[i])) for i in range(2)]
    bs = [rng.uniform(-.5, .5, widths[i + 1]) for i in range(2)]
    gamma, beta = 0.1 * rng.standard_normal(16), 0.1 * rng.standard_normal(16)
    alpha = rng.uniform(0.5, 3, nout)
    idx = np.arange(S ** 3)
    out = oracle.filter_gen_3d_points(g, False, F, Ws, bs, gamma, beta, alpha, idx)
    ix, iy, iz = idx // (S * S), (idx // S) % S, idx % S
    r = np.stack([np.where(a < S // 2, a, a - S) for a in (ix, iy, iz)], axis=1)
    inside = np.all(np.abs(r) <= g - 1, axis=1)
    # the index S/2 on any axis (offset -g) is outside the support
    assert not inside[(ix == S // 2) | (iy == S // 2) | (iz == S // 2)].any()
    jj = np.arange(1, F + 1)
    feats = []
    for a in range(3):
        ang = np.pi * np.outer(r[:, a], jj) / g
        feats += [np.cos(ang), np.sin(ang)]
    pe = np.concatenate(feats, axis=1)
    rn = np.sqrt((r.astype(float) ** 2).sum(1)) / g
    ref = _np_mlp(pe, Ws, bs, gamma, beta) * np.exp(-np.outer(rn, alpha))
    ref[~inside] = 0
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # circular grid: every index is in the support
    outc = oracle.filter_gen_3d_points(g, True, F, Ws, bs, gamma, beta, alpha, np.arange(g ** 3))
    assert np.all(np.abs(outc).sum(1) > 0)


# ---------------------------------------------------------------- a3 spectrum

def test_dft_real_rows():
    L, n = 16, 32
    h = np.zeros((3, L))
    h[0, 0] = 1.0
    h[1, 5] = 2.0
    h[2] = np.random.default_rng(3).standard_normal(L)
    H = oracle.dft_real_rows(h, n)
    k = np.arange(n // 2 + 1)
    np.testing.assert_allclose(H[0], np.ones(n // 2 + 1), atol=1e-15)
    np.testing.assert_allclose(H[1], 2 * np.exp(-2j * np.pi * k * 5 / n), atol=1e-14)
    np.testing.assert_allclose(H, np.fft.rfft(h, n=n, axis=-1), atol=1e-12)


# ---------------------------------------------------------------- a4-a7 causal conv

def test_causal_conv_delta_and_skip():
    u = np.random.default_rng(4).standard_normal(50)
    h = np.zeros(50); h[0] = 1.0
    np.testing.assert_array_equal(oracle.causal_conv(h, u), u)
    np.testing.assert_allclose(oracle.causal_conv(h, u, 0.25), 1.25 * u, rtol=1e-15)


def test_causal_conv_geometric_closed_form():
    L = 300
    rho = math.exp(-2.0 / L)
    h = rho ** np.arange(L)
    c = oracle.causal_conv(h, np.ones(L))
    t = np.arange(L)
    np.testing.assert_allclose(c, (1 - rho ** (t + 1)) / (1 - rho), rtol=1e-12)
    # first-order recurrence for any input
    u = np.random.default_rng(5).standard_normal(L)
    c = oracle.causal_conv(h, u)
    np.testing.assert_allclose(c[1:], rho * c[:-1] + u[1:], rtol=1e-10, atol=1e-12)
    assert c[0] == u[0]


def test_causal_conv_linearity_and_shift():
    rng = np.random.default_rng(6)
    L = 64
    h, h2, u1, u2 = rng.standard_normal((4, L))
    a, b = 1.5, -0.75
    np.testing.assert_allclose(oracle.causal_conv(h, a * u1 + b * u2),
                               a * oracle.causal_conv(h, u1) + b * oracle.causal_conv(h, u2),
                               atol=1e-12)
    np.testing.assert_allclose(oracle.causal_conv(a * h + b * h2, u1),
                               a * oracle.causal_conv(h, u1) + b * oracle.causal_conv(h2, u1),
                               atol=1e-12)
    s = 7
    us = np.r_[np.zeros(s), u1[:-s]]
    np.testing.assert_allclose(oracle.causal_conv(h, us)[s:], oracle.causal_conv(h, u1)[:-s],
                               atol=1e-12)
    assert np.all(oracle.causal_conv(h, us)[:s] == 0)


@pytest.mark.parametrize("L", [1, 2, 5, 16, 33, 64])
def test_causal_conv_bruteforce_toeplitz(L):
    rng = np.random.default_rng(L)
    h = rng.integers(-4, 5, L).astype(float)
    u = rng.integers(-4, 5, L).astype(float)
    T = np.zeros((L, L))
    for i in range(L):
        for j in range(i + 1):
            T[i, j] = h[i - j]
    np.testing.assert_array_equal(oracle.causal_conv(h, u, 3.0), T @ u + 3.0 * u)


def test_golden_causal_conv_gate():
    gd = _golden("causal_conv_gate_L4.json")
    c = oracle.causal_conv(gd["h"], gd["v"], gd["D"])
    np.testing.assert_array_equal(c, gd["c"])
    v = np.array(gd["v"], float).reshape(1, 1, 4)
    x1 = np.array(gd["x1"], float).reshape(1, 1, 4)
    h = np.array(gd["h"], float).reshape(1, 1, 4)
    y = oracle.hyena_rows(v, [x1], h, np.array([[gd["D"]]]))
    np.testing.assert_array_equal(y[0], gd["y"])


def test_chain_reductions():
    rng = np.random.default_rng(7)
    B, D, L = 2, 3, 40
    v = rng.standard_normal((B, D, L))
    h = rng.standard_normal((2, D, L))
    Dk = rng.standard_normal((2, D))
    ones = np.ones((B, D, L))
    # order 2 with x1 = 1 is the convolution plus skip
    y = oracle.hyena_rows(v, [ones], h[:1], Dk[:1])
    for b in range(B):
        for d in range(D):
            np.testing.assert_allclose(y[b * D + d], oracle.causal_conv(h[0, d], v[b, d], Dk[0, d]),
                                       rtol=0, atol=0)
    # order 3 with a delta filter at order 2: y = x2 * (1 + D_2) * z1
    x1 = rng.standard_normal((B, D, L)); x2 = rng.standard_normal((B, D, L))
    hd = h.copy(); hd[1] = 0; hd[1, :, 0] = 1
    z1 = oracle.hyena_rows(v, [x1], h[:1], Dk[:1]).reshape(B, D, L)
    y3 = oracle.hyena_rows(v, [x1, x2], hd, Dk).reshape(B, D, L)
    np.testing.assert_allclose(y3, x2 * (1 + Dk[1][None, :, None]) * z1, rtol=1e-14, atol=1e-14)
    # no skip at all
    y0 = oracle.hyena_rows(v, [ones], h[:1], None)
    np.testing.assert_array_equal(y0[0], oracle.causal_conv(h[0, 0], v[0, 0]))
    # a prefix of the chain depends only on prefixes
    yp = oracle.hyena_rows(v, [x1, x2], h, Dk, rows=[4], T=17)
    np.testing.assert_array_equal(yp[0], oracle.hyena_rows(v, [x1, x2], h, Dk)[4, :17])


@pytest.mark.parametrize("L", [3, 16, 64])
def test_chain_bruteforce(L):
    rng = np.random.default_rng(100 + L)
    K, D = 3, 2
    ints = lambda *s: rng.integers(-2, 3, s).astype(float)
    v, xs, h, Dk = ints(1, D, L), [ints(1, D, L) for _ in range(K)], ints(K, D, L), ints(K, D)
    y = oracle.hyena_rows(v, xs, h, Dk)
    for d in range(D):
        z = v[0, d]
        for k in range(K):
            T = np.array([[h[k, d, i - j] if j <= i else 0.0 for j in range(L)] for i in range(L)])
            z = xs[k][0, d] * (T @ z + Dk[k, d] * z)
        np.testing.assert_array_equal(y[d], z)


def test_conv_gate_samples_match_rows():
    rng = np.random.default_rng(8)
    L = 200
    h, u, x = rng.standard_normal((3, L))
    ts = np.array([0, 1, 57, 199])
    s = oracle.conv_gate_samples(h, u, x, 0.3, ts)
    full = oracle.hyena_rows(u.reshape(1, 1, L), [x.reshape(1, 1, L)], h.reshape(1, 1, L), np.array([[0.3]]))
    np.testing.assert_allclose(s, full[0, ts], rtol=0, atol=0)


# ---------------------------------------------------------------- a9 N-D

def _nd_brute(K, v, circular):
    g = v.shape
    S = g if circular else tuple(2 * a for a in g)
    c = np.zeros(g)
    for p in np.ndindex(*g):
        s = 0.0
        for q in np.ndindex(*g):
            s += K[tuple((p[a] - q[a]) % S[a] for a in range(3))] * v[q]
        c[p] = s
    return c


def test_golden_nd():
    gd = _golden("nd_conv_2cube.json")
    g = tuple(gd["g"])
    K = np.zeros(tuple(2 * a for a in g))
    for i, j, l, val in gd["kernel_entries"]:
        K[int(i), int(j), int(l)] = val
    v = np.array(gd["v"], float)
    pts = np.arange(int(np.prod(g)))
    c = oracle.nd_conv_points(K, v, None, 0.0, pts).reshape(g)
    np.testing.assert_array_equal(c, gd["c"])


@pytest.mark.parametrize("circular", [False, True])
def test_nd_bruteforce_and_delta(circular):
    rng = np.random.default_rng(9)
    g = (3, 4, 2)
    S = g if circular else tuple(2 * a for a in g)
    K = rng.standard_normal(S)
    v, x1 = rng.standard_normal((2,) + g)
    pts = np.arange(int(np.prod(g)))
    y = oracle.nd_conv_points(K, v, x1, 0.5, pts, circular).reshape(g)
    np.testing.assert_allclose(y, x1 * (_nd_brute(K, v, circular) + 0.5 * v), rtol=1e-13, atol=1e-13)
    Kd = np.zeros(S); Kd[0, 0, 0] = 1
    np.testing.assert_array_equal(oracle.nd_conv_points(Kd, v, x1, 0.0, pts, circular).reshape(g), x1 * v)


def test_nd_separable():
    rng = np.random.default_rng(10)
    g = 5
    S = 2 * g
    ks = [rng.standard_normal(2 * g - 1) for _ in range(3)]   # offsets -(g-1)..(g-1)
    vs = [rng.standard_normal(g) for _ in range(3)]
    K = np.zeros((S, S, S))
    for a in range(-(g - 1), g):
        for b in range(-(g - 1), g):
            for c in range(-(g - 1), g):
                K[a % S, b % S, c % S] = ks[0][a + g - 1] * ks[1][b + g - 1] * ks[2][c + g - 1]
    v = np.einsum("i,j,k->ijk", *vs)
    y = oracle.nd_conv_points(K, v, None, 0.0, np.arange(g ** 3)).reshape(g, g, g)
    one_d = [np.convolve(ks[a], vs[a])[g - 1: 2 * g - 1] for a in range(3)]
    np.testing.assert_allclose(y, np.einsum("i,j,k->ijk", *one_d), rtol=1e-12, atol=1e-12)


def test_nd_shift_equivariance():
    rng = np.random.default_rng(11)
    g = (6, 6, 6)
    K = rng.standard_normal((12, 12, 12))
    v = np.zeros(g); v[:4, :4, :4] = rng.standard_normal((4, 4, 4))
    vs = np.zeros(g); vs[2:, 1:5, 2:] = v[:4, :4, :4]
    pts = np.arange(216)
    a = oracle.nd_conv_points(K, v, None, 0.0, pts).reshape(g)
    b = oracle.nd_conv_points(K, vs, None, 0.0, pts).reshape(g)
    np.testing.assert_allclose(b[2:, 1:, 2:], a[:4, :5, :4], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- a10 spectral gate

def test_golden_spectral_gate():
    gd = _golden("spectral_gate_n4.json")
    g = np.array(gd["g_re"]) + 1j * np.array(gd["g_im"])
    kap = oracle.gate_kernel(g)
    mixed = oracle.circular_conv_samples(kap, gd["x1"], None, np.arange(4))
    np.testing.assert_allclose(mixed, gd["mixed"], atol=1e-14)
    y = oracle.circular_conv_samples(kap, gd["x1"], gd["x2"], np.arange(4))
    np.testing.assert_allclose(y, gd["y"], atol=1e-14)


def test_gate_kernel_special_cases():
    n = 64
    nb = n // 2 + 1
    k = np.arange(nb)
    kap = oracle.gate_kernel(np.ones(nb))
    np.testing.assert_allclose(kap, np.r_[1.0, np.zeros(n - 1)], atol=1e-14)
    for s in (1, 5, 32, 63):
        kap = oracle.gate_kernel(np.exp(-2j * np.pi * k * s / n))
        e = np.zeros(n); e[s] = 1
        np.testing.assert_allclose(kap, e, atol=1e-13)
    kap = oracle.gate_kernel(np.full(nb, -1.75 + 0j))
    np.testing.assert_allclose(kap, np.r_[-1.75, np.zeros(n - 1)], atol=1e-14)
    rng = np.random.default_rng(12)
    g = rng.standard_normal(nb) + 1j * rng.standard_normal(nb)
    np.testing.assert_allclose(oracle.gate_kernel(g), np.fft.irfft(g, n=n), atol=1e-13)


def test_circular_conv_shift_parseval_library():
    rng = np.random.default_rng(13)
    n = 32
    x1 = rng.standard_normal(n)
    s = 3
    e = np.zeros(n); e[s] = 1
    y = oracle.circular_conv_samples(e, x1, None, np.arange(n))
    np.testing.assert_array_equal(y, np.roll(x1, s))
    kap = rng.standard_normal(n)
    y = oracle.circular_conv_samples(kap, x1, None, np.arange(n))
    G, X = np.fft.fft(kap), np.fft.fft(x1)
    np.testing.assert_allclose(np.sum(y ** 2), np.sum(np.abs(G * X) ** 2) / n, rtol=1e-12)
    np.testing.assert_allclose(y, np.real(np.fft.ifft(G * X)), atol=1e-12)
    rows = oracle.circular_conv_rows(np.stack([kap, e]), [1, 0], np.stack([x1, x1]), None)
    np.testing.assert_array_equal(rows[0], np.roll(x1, s))
    np.testing.assert_allclose(rows[1], y, atol=1e-13)


# ---------------------------------------------------------------- FFT-route references

def test_fft_hyena_rows_matches_direct():
    rng = np.random.default_rng(14)
    B, D, L = 2, 3, 100            # L not a power of two: padded transform 256
    v = rng.standard_normal((B, D, L))
    xs = [rng.standard_normal((B, D, L)) for _ in range(2)]
    h = rng.standard_normal((2, D, L)) * np.exp(-np.arange(L) / 30)
    Dk = rng.standard_normal((2, D))
    a = oracle.fft_hyena_rows(v, xs, h, Dk)
    b = oracle.hyena_rows(v, xs, h, Dk)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)
    assert oracle.transform_len(100) == 256 and oracle.transform_len(128) == 256


def test_fft_nd_matches_direct():
    rng = np.random.default_rng(15)
    g = (4, 6, 8)
    for circular in (False, True):
        S = g if circular else tuple(2 * a for a in g)
        K = rng.standard_normal(S)
        v, x1 = rng.standard_normal((2,) + g)
        a = oracle.fft_nd_conv(K, v, x1, 0.2, circular)
        b = oracle.nd_conv_points(K, v, x1, 0.2, np.arange(int(np.prod(g))), circular).reshape(g)
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)


def test_fft_spectral_gate_matches_direct():
    rng = np.random.default_rng(16)
    n, R = 64, 3
    g = rng.standard_normal((2, n // 2 + 1)) + 1j * rng.standard_normal((2, n // 2 + 1))
    x1, x2 = rng.standard_normal((2, R, n))
    kidx = np.array([0, 1, 1])
    a = oracle.fft_spectral_gate_rows(g[kidx], x1, x2)
    kap = np.stack([oracle.gate_kernel(gg) for gg in g])
    b = oracle.circular_conv_rows(kap, kidx, x1, x2)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_fft_spectrum_matches_direct():
    rng = np.random.default_rng(17)
    h = rng.standard_normal((4, 40))
    np.testing.assert_allclose(oracle.fft_spectrum(h), oracle.dft_real_rows(h, 128), atol=1e-11)


# ---------------------------------------------------------------- naive CPU FFT reference

def test_fftref_fft_closed_forms_and_direct_dft():
    """The naive radix-2 FFT: a delta at s transforms to the phase ramp
    e^{-2 pi i k s/n} (closed form), a constant c to n c at k = 0 and zeros
    elsewhere, inverse(forward(x)) = n x, and a real row equals the direct
    DFT of hyena_oracle.c (not numpy) on every bin."""
    n = 64
    k = np.arange(n)
    for s in (0, 1, 5, 32, 63):
        e = np.zeros(n, complex)
        e[s] = 1.0
        np.testing.assert_allclose(oracle.fftref_fft(e), np.exp(-2j * np.pi * k * s / n), atol=1e-14)
        np.testing.assert_allclose(oracle.fftref_fft(e, inverse=True), np.exp(2j * np.pi * k * s / n), atol=1e-14)
    c = np.full(n, 0.75 - 0.5j)
    X = oracle.fftref_fft(c)
    np.testing.assert_allclose(X[0], n * (0.75 - 0.5j), atol=1e-13)
    np.testing.assert_allclose(X[1:], 0, atol=1e-13)
    rng = np.random.default_rng(40)
    x = rng.standard_normal(n) + 1j * rng.standard_normal(n)
    np.testing.assert_allclose(oracle.fftref_fft(oracle.fftref_fft(x), inverse=True), n * x, atol=1e-12)
    h = rng.standard_normal((3, 40))
    for r in range(3):
        pad = np.zeros(128, complex)
        pad[:40] = h[r]
        np.testing.assert_allclose(oracle.fftref_fft(pad)[:65], oracle.dft_real_rows(h[r:r + 1], 128)[0],
                                   atol=1e-12)


def test_fftref_hyena_rows_matches_direct():
    rng = np.random.default_rng(41)
    for (B, D, L, K) in [(2, 3, 100, 1), (1, 2, 64, 3), (1, 1, 1, 2)]:
        v = rng.standard_normal((B, D, L))
        xs = [rng.standard_normal((B, D, L)) for _ in range(K)]
        h = rng.standard_normal((K, D, L)) * np.exp(-np.arange(L) / 30)
        Dk = rng.standard_normal((K, D))
        a = oracle.fftref_hyena_rows(v, xs, h, Dk)
        b = oracle.hyena_rows(v, xs, h, Dk)
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-11)
    rows = np.array([4, 0])
    a = oracle.fftref_hyena_rows(v, xs, h, None, rows=rows)
    np.testing.assert_allclose(a, oracle.hyena_rows(v, xs, h, None, rows=rows), rtol=1e-10, atol=1e-11)


def test_fftref_gate_and_nd_match_direct():
    rng = np.random.default_rng(42)
    n = 64
    g = rng.standard_normal((2, n // 2 + 1)) + 1j * rng.standard_normal((2, n // 2 + 1))
    x1, x2 = rng.standard_normal((2, 3, n))
    gidx = np.array([1, 0, 1])
    kap = np.stack([oracle.gate_kernel(gg) for gg in g])
    np.testing.assert_allclose(oracle.fftref_gate_rows(g, gidx, x1, x2),
                               oracle.circular_conv_rows(kap, gidx, x1, x2), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(oracle.fftref_gate_rows(g, gidx, x1, None),
                               oracle.circular_conv_rows(kap, gidx, x1, None), rtol=1e-11, atol=1e-12)
    gr = (4, 2, 8)
    for circular in (False, True):
        S = gr if circular else tuple(2 * a for a in gr)
        Kern = rng.standard_normal((2,) + S)
        v, x1 = rng.standard_normal((2, 3) + gr)
        kidx = np.array([1, 1, 0])
        a = oracle.fftref_nd_conv(Kern, kidx, v, x1, circular)
        for s in range(3):
            b = oracle.nd_conv_points(Kern[kidx[s]], v[s], x1[s], 0.0, np.arange(int(np.prod(gr))),
                                      circular).reshape(gr)
            np.testing.assert_allclose(a[s], b, rtol=1e-11, atol=1e-11)


# ---------------------------------------------------------------- HyenaND register conditioning

def test_register_film_closed_forms():
    """z(x) = softmax-weighted mean of the register activations
    ([ND] 레지스터 및 FiLM): without logits it is the plain mean; a logit far
    above the rest selects that register; adding a constant to every logit of
    a sample changes nothing; logits of 1e4 stay finite (the maximum is
    subtracted); the FiLM map with identity blocks returns z and with zero
    weights the bias."""
    rng = np.random.default_rng(50)
    B, R, C, H = 3, 5, 6, 6
    reg = rng.standard_normal((B, R, C))
    I = np.eye(C)
    W = np.concatenate([I, 2 * I])
    b0 = np.zeros(2 * H)
    g, be, z, w = oracle.register_film(reg, None, None, W, b0)
    np.testing.assert_allclose(z, reg.mean(axis=1), rtol=0, atol=1e-15)
    np.testing.assert_allclose(g, z, atol=1e-15)
    np.testing.assert_allclose(be, 2 * z, atol=1e-15)
    s = np.zeros((B, R))
    s[np.arange(B), [4, 0, 2]] = 60.0
    _, _, z1, _ = oracle.register_film(reg, None, s, W, b0)
    np.testing.assert_allclose(z1, reg[np.arange(B), [4, 0, 2]], atol=1e-12)
    s2 = rng.standard_normal((B, R))
    _, _, za, _ = oracle.register_film(reg, None, s2, W, b0)
    _, _, zb, _ = oracle.register_film(reg, None, s2 + rng.standard_normal((B, 1)) * 100, W, b0)
    np.testing.assert_allclose(za, zb, rtol=1e-12, atol=1e-13)
    _, _, zc, wc = oracle.register_film(reg, None, 1e4 * s2, W, b0)
    assert np.all(np.isfinite(zc)) and np.allclose(wc.sum(axis=1), 1.0)
    c = rng.standard_normal(2 * H)
    g0, be0, _, _ = oracle.register_film(reg, rng.standard_normal(C), s2, np.zeros((2 * H, C)), c)
    np.testing.assert_array_equal(g0, np.broadcast_to(c[:H], (B, H)))
    np.testing.assert_array_equal(be0, np.broadcast_to(c[H:], (B, H)))


def test_register_film_bruteforce_loops():
    """Query logits and FiLM map against plain Python loops on a tiny case."""
    rng = np.random.default_rng(51)
    B, R, C, H = 2, 3, 4, 2
    reg = rng.standard_normal((B, R, C))
    q = rng.standard_normal(C)
    sc = rng.standard_normal((B, R))
    W = rng.standard_normal((2 * H, C))
    bb = rng.standard_normal(2 * H)
    g, be, z, w = oracle.register_film(reg, q, sc, W, bb)
    for bi in range(B):
        lg = [sum(q[c] * reg[bi, r, c] for c in range(C)) + sc[bi, r] for r in range(R)]
        ex = [math.exp(v) for v in lg]
        tot = sum(ex)
        zz = [sum(ex[r] / tot * reg[bi, r, c] for r in range(R)) for c in range(C)]
        out = [bb[o] + sum(W[o, c] * zz[c] for c in range(C)) for o in range(2 * H)]
        np.testing.assert_allclose(z[bi], zz, rtol=1e-12)
        np.testing.assert_allclose(g[bi], out[:H], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(be[bi], out[H:], rtol=1e-12, atol=1e-14)


def test_projection_identity_zero_and_linearity():
    """Input projection: identity blocks return the input transposed to
    channel-major (times the block's scale), zero weights return the bias on
    every position, and the map is linear in x."""
    rng = np.random.default_rng(18)
    B, L, C = 2, 7, 5
    x = rng.standard_normal((B, L, C))
    W = np.concatenate([np.eye(C), 3.0 * np.eye(C)])          # n_out = 2, D = C
    v, x1 = oracle.projection(x, W, None, 2)
    assert v.shape == (B, C, L)
    np.testing.assert_array_equal(v, x.transpose(0, 2, 1))
    np.testing.assert_array_equal(x1, 3.0 * x.transpose(0, 2, 1))
    bias = rng.standard_normal(3 * 4)
    outs = oracle.projection(x, np.zeros((12, C)), bias, 3)
    for k, o in enumerate(outs):
        np.testing.assert_array_equal(o, np.broadcast_to(bias[4 * k:4 * k + 4][None, :, None], (B, 4, L)))
    W2 = rng.standard_normal((8, C))
    x2 = rng.standard_normal((B, L, C))
    a = oracle.projection(x + 2 * x2, W2, None, 2)
    b1, b2 = oracle.projection(x, W2, None, 2), oracle.projection(x2, W2, None, 2)
    for k in range(2):
        np.testing.assert_allclose(a[k], b1[k] + 2 * b2[k], rtol=1e-12, atol=1e-12)


def test_backward_matches_finite_differences():
    """Every gradient of the float64 backward equals the central difference of
    the loss sum(dy * y), with y from the direct forward oracle (the C
    hyena_rows, a separate code path), at a few elements of each input."""
    rng = np.random.default_rng(19)
    B, D, L, K = 2, 3, 11, 2
    v = rng.standard_normal((B, D, L))
    xs = [rng.standard_normal((B, D, L)) for _ in range(K)]
    h = rng.standard_normal((K, D, L)) * 0.5
    Dk = rng.standard_normal((K, D))
    dy = rng.standard_normal((B, D, L))
    dv, dxs, dh, dD = oracle.hyena_backward(v, xs, h, Dk, dy)

    def loss(v_, xs_, h_, D_):
        return float(np.sum(dy * oracle.hyena_rows(v_, xs_, h_, D_).reshape(B, D, L)))

    eps = 1e-6

    def fd(make):
        return (loss(*make(eps)) - loss(*make(-eps))) / (2 * eps)

    for i in [(0, 0, 0), (1, 2, 5), (0, 1, L - 1)]:
        def mv(e, i=i):
            a = v.copy(); a[i] += e
            return a, xs, h, Dk
        assert abs(fd(mv) - dv[i]) < 1e-6 * (1 + abs(dv[i]))
        for k in range(K):
            def mx(e, i=i, k=k):
                a = [x.copy() for x in xs]; a[k][i] += e
                return v, a, h, Dk
            assert abs(fd(mx) - dxs[k][i]) < 1e-6 * (1 + abs(dxs[k][i]))
    for k in range(K):
        for j in [(0, 0), (2, 4), (1, L - 1)]:
            def mh(e, j=j, k=k):
                a = h.copy(); a[(k,) + j] += e
                return v, xs, a, Dk
            assert abs(fd(mh) - dh[(k,) + j]) < 1e-6 * (1 + abs(dh[(k,) + j]))
        for d in range(D):
            def md(e, d=d, k=k):
                a = Dk.copy(); a[k, d] += e
                return v, xs, h, a
            assert abs(fd(md) - dD[k, d]) < 1e-6 * (1 + abs(dD[k, d]))


def test_backward_samples_equal_full_backward():
    rng = np.random.default_rng(20)
    B, D, L = 2, 3, 40
    v, x1, dy = rng.standard_normal((3, B, D, L))
    h = rng.standard_normal((D, L))
    Dk = rng.standard_normal(D)
    dv, dxs, dh, dD = oracle.hyena_backward(v, [x1], h[None], Dk[None], dy)
    ts = np.arange(L)
    sv, sx, sh, sD = oracle.hyena_backward_samples(v, x1, h, Dk, dy, ts)
    np.testing.assert_allclose(sv, dv, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sx, dxs[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sh, dh[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sD, dD[0], rtol=1e-12, atol=1e-12)


def test_filter_gen_sine_and_gaussian_window_closed_forms():
    """SIREN hidden layers with frequency 0 output sin(0) = 0, so the filter
    is the last bias under the window: b_o exp(-alpha_o n^2) for the Gaussian
    window (n = t/L in 1-D, |r|/g in 3-D); the identity activation makes the
    MLP one affine map of the encoding."""
    rng = np.random.default_rng(23)
    L, F, nout = 64, 4, 3
    Ws = [rng.standard_normal((16, 9)), rng.standard_normal((8, 16)), rng.standard_normal((nout, 8))]
    bs = [rng.standard_normal(16), rng.standard_normal(8), rng.standard_normal(nout)]
    alpha = rng.uniform(0.5, 3.0, nout)
    h = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act="sine", omega=np.zeros(24), window="gauss")
    n = np.arange(L) / L
    np.testing.assert_allclose(h, bs[2][:, None] * np.exp(-alpha[:, None] * n[None] ** 2), rtol=1e-14, atol=1e-14)
    g = 4
    Ws3 = [rng.standard_normal((16, 6 * 2)), rng.standard_normal((nout, 16))]
    bs3 = [rng.standard_normal(16), rng.standard_normal(nout)]
    idx = np.arange((2 * g) ** 3)
    pts = oracle.filter_gen_3d_points(g, False, 2, Ws3, bs3, rng.standard_normal(16) * 0.1,
                                      rng.standard_normal(16) * 0.1, alpha, idx, act="sine",
                                      omega=np.zeros(16), window="gauss")
    S = 2 * g
    off = lambda i: np.where(i < S // 2, i, i - S)
    r = np.stack([off(idx // (S * S)), off((idx // S) % S), off(idx % S)], 1)
    inside = np.all(np.abs(r) < g, 1)
    rn2 = np.sum(r.astype(np.float64) ** 2, 1) / g ** 2
    ref = np.where(inside[:, None], bs3[1][None] * np.exp(-alpha[None] * rn2[:, None]), 0.0)
    np.testing.assert_allclose(pts, ref, rtol=1e-14, atol=1e-14)
    lin = oracle.filter_gen_1d(L, F, True, Ws, bs, alpha, act="identity")
    pe = oracle.pe1d(L, F, True)
    aff = ((pe @ Ws[0].T + bs[0]) @ Ws[1].T + bs[1]) @ Ws[2].T + bs[2]
    np.testing.assert_allclose(lin, aff.T * np.exp(-alpha[:, None] * n[None]), rtol=1e-11, atol=1e-11)


def test_prefix_gate_outputs_first_step_and_full_prefix():
    """Streaming gate: the first output is x2[0] kappa[0] x[0]; the last one
    (whole sequence seen) equals the full circular convolution there."""
    rng = np.random.default_rng(24)
    n = 32
    g = rng.standard_normal(n // 2 + 1) + 1j * rng.standard_normal(n // 2 + 1)
    x1, x2 = rng.standard_normal((2, n))
    out = oracle.prefix_gate_outputs(g, x1, x2, n)
    kap = oracle.gate_kernel(g)
    assert abs(out[0] - x2[0] * kap[0] * x1[0]) < 1e-12
    full = oracle.circular_conv_samples(kap, x1, x2, [n - 1])[0]
    assert abs(out[-1] - full) < 1e-12
