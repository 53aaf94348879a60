"""Float64 CPU oracle for the Hyena hot path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
this package imports nothing from the product package: the two share no
code.  Inputs come from ``hyena_workloads`` (random draws only).

Two layers:

* ``hyena_oracle.c`` (compiled here with gcc, float64, OpenMP over rows): the
  plain definitions -- direct O(L^2) causal convolution and gating chain,
  direct N-D convolution, direct DFTs, the filter MLP.
* FFT-route references below (``fft_*``): the same quantities through
  ``numpy.fft`` in float64, used as a library step, for tensors too large for
  the direct sums.  They are trusted only where the tests have matched them
  against the direct definitions.
* ``fft_reference.c`` (``fftref_*``): a naive float64 CPU FFT route (one
  iterative radix-2 complex FFT, real rows as complex, the filter transform
  recomputed per row) -- the plain CPU program the benchmark times beside the
  direct oracle.  Pinned to the direct definitions like the ``fft_*`` ones.

Pages cited (title, section):
  [HN] "Hyena: 암묵적 장거리 컨볼루션으로 어텐션을 완전 대체한 서브-이차 모델",
       아키텍처 상세 (steps 1, 2 and 3) and its ImplicitFilter / hyena_operator sketch.
  [ES] "4. Hyena 상세", 어떻게 동작하나요?.
  [ND] "Native Multi-Dimensional Subquadratic Operators via Input Dependent Long
       Convolutions", 방법론: HyenaND (네이티브 ND 합성곱, 경계 처리).
  [SP] "FFT의 반격: Self-Attention의 효율적 대안", 토큰 믹서 구성과 생성 지원.

Parity status per function is listed in ``PINS`` (every function is pinned by
a test in ``tests/test_oracle_pins.py``; none is "parity unpinned").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_SRC_FFT = os.path.join(_HERE, "fft_reference.c")
_BUILD = os.path.join(_HERE, "_build")
_SO = os.path.join(_BUILD, "libhyena_oracle.so")

PINS = {
    "pe1d": "closed forms at t=0 and t=L/4; numpy cos/sin",
    "filter_gen_1d": "constant-output MLP; numpy float64 matmul MLP",
    "filter_gen_3d_points": "support mask, zero offset, numpy float64 matmul MLP",
    "dft_real_rows": "delta filter closed form; numpy.fft.rfft",
    "causal_conv": "delta, geometric closed form, recurrence, linearity, shift, Toeplitz brute force",
    "hyena_rows": "x=1 reduction, delta-filter reduction, brute force on L<=64",
    "conv_gate_samples": "equals hyena_rows order 1",
    "nd_conv_points": "delta kernel, separable product of 1-D convolutions, shift, brute force, circular wrap",
    "gate_kernel": "g=1 delta, shift gate, constant gate, numpy.fft.irfft",
    "circular_conv": "shift gate, Parseval, numpy.fft circular convolution",
    "fft_*": "matched against the direct functions above on sampled outputs",
    "fftref_fft": "delta and constant closed forms, inverse(forward) = n x, direct DFT (dft_real_rows)",
    "fftref_*": "equal to the direct hyena_rows, gate kernel + circular_conv_rows and nd_conv_points",
    "projection": "identity weights give the transposed input, zero weights the bias, linearity",
    "register_film": "no logits -> plain mean, one-hot limit -> selection, shift invariance, stable at large "
                     "logits, loop brute force, identity / zero FiLM maps",
    "hyena_backward": "central finite differences of the direct forward (hyena_rows) for every input",
    "hyena_backward_samples": "equals hyena_backward (order 2) at every index",
    "prefix_gate_outputs": "composition of gate_kernel and circular_conv_samples (pinned); first output x2 kappa[0] x",
}


def build(force: bool = False) -> str:
    """Compile hyena_oracle.c and fft_reference.c into
    oracle/_build/libhyena_oracle.so (gcc)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_SO)
            and os.path.getmtime(_SO) >= max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_FFT))):
        return _SO
    tmp = _SO + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
           _SRC, _SRC_FFT, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _SO)
    return _SO


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
    return _lib


_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def _dp(a: np.ndarray):
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(_D)


def _ip(a: np.ndarray):
    assert a.dtype == np.int64 and a.flags.c_contiguous
    return a.ctypes.data_as(_I64)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr_array(arrs: Sequence[np.ndarray]):
    arr = (_D * len(arrs))()
    for i, a in enumerate(arrs):
        arr[i] = _dp(a)
    return arr


def threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else the affinity set)."""
    env = os.environ.get("OMP_NUM_THREADS")
    return int(env) if env else len(os.sched_getaffinity(0))


# --------------------------------------------------------------------------
# input projection ([HN] 아키텍처 상세, step 1: v, x_1, ... = split(W_proj x))
# --------------------------------------------------------------------------

def projection(x, W, bias, n_out: int) -> list:
    """out_k[b, d, l] = bias[kD + d] + sum_c W[kD + d, c] x[b, l, c], float64.

    x: (B, L, C); W: (n_out*D, C); bias: (n_out*D,) or None.  Returns the
    n_out channel-major (B, D, L) arrays (the split of W_proj x)."""
    x = np.asarray(x, np.float64)
    W = np.asarray(W, np.float64)
    D = W.shape[0] // n_out
    assert W.shape[0] == n_out * D and W.shape[1] == x.shape[2]
    full = np.matmul(x, W.T)                        # (B, L, n_out*D), a library matmul
    if bias is not None:
        full = full + np.asarray(bias, np.float64)[None, None, :]
    return [np.ascontiguousarray(full[:, :, k * D:(k + 1) * D].transpose(0, 2, 1)) for k in range(n_out)]


# --------------------------------------------------------------------------
# HyenaND input conditioning ([ND] 방법론: HyenaND, 레지스터 및 FiLM을 통한 입력
# 의존적 커널): register activations -> z(x) by a softmax-weighted mean ->
# FiLM parameters of the kernel MLP
# --------------------------------------------------------------------------

def register_film(reg, query, scores, W, b):
    """z(x) and the FiLM parameters it drives, float64.

    reg: (B, R, C) activations of the R register tokens of each sample.
    Pooling logits l[b, r] = query . reg[b, r] (if query is given) + scores[b, r]
    (if given); weights w[b] = softmax_r(l[b]); z[b] = sum_r w[b, r] reg[b, r].
    The control variable drives FiLM through one linear map:
    (gamma[b], beta[b]) = W z[b] + b, W of shape (2 H, C), gamma the first H
    outputs and beta the next H.  Returns (gamma, beta, z, w)."""
    reg = np.asarray(reg, np.float64)
    B, R, C = reg.shape
    logits = np.zeros((B, R))
    if query is not None:
        logits = logits + np.einsum("brc,c->br", reg, np.asarray(query, np.float64))
    if scores is not None:
        logits = logits + np.asarray(scores, np.float64)
    m = logits.max(axis=1, keepdims=True)           # softmax with the maximum subtracted
    e = np.exp(logits - m)
    w = e / e.sum(axis=1, keepdims=True)
    z = np.einsum("br,brc->bc", w, reg)
    out = z @ np.asarray(W, np.float64).T + np.asarray(b, np.float64)[None, :]
    H = out.shape[1] // 2
    return out[:, :H], out[:, H:], z, w


# --------------------------------------------------------------------------
# a1 / a2: positional encoding and filter MLP
# --------------------------------------------------------------------------

def pe1d(L: int, F: int, include_t: bool = True) -> np.ndarray:
    w = int(include_t) + 2 * F
    out = np.empty((L, w), np.float64)
    _load().orc_pe1d(ctypes.c_int64(L), ctypes.c_int(F), ctypes.c_int(int(include_t)), _dp(out))
    return out


def _mlp_args(Ws, bs):
    Ws = [_f64(w) for w in Ws]
    bs = [_f64(b) for b in bs]
    widths = [Ws[0].shape[1]] + [w.shape[0] for w in Ws]
    for l, w in enumerate(Ws):
        assert w.shape == (widths[l + 1], widths[l]) and bs[l].shape == (widths[l + 1],)
    warr = (ctypes.c_int * len(widths))(*widths)
    return Ws, bs, widths, warr


ACT = {"silu": 0, "identity": 1, "sine": 2}
WINDOW = {"exp": 0, "gauss": 1}


def _omega_arg(omega, widths):
    """Per-hidden-unit sine frequencies, all hidden layers concatenated."""
    if omega is None:
        return None, None
    om = _f64(omega)
    assert om.shape == (sum(widths[1:-1]),)
    return om, _dp(om)


def filter_gen_1d(L, F, include_t, Ws, bs, alpha, act="silu", omega=None, window="exp") -> np.ndarray:
    """h[o, t] = MLP(PE(t))[o] * w_o(t/L), float64, shape (n_out, L); hidden
    activation SiLU, identity or sin(omega x); window exp(-alpha_o n) or the
    Gaussian exp(-alpha_o n^2)."""
    Ws, bs, widths, warr = _mlp_args(Ws, bs)
    alpha = _f64(alpha)
    nout = widths[-1]
    assert alpha.shape == (nout,)
    om, omp = _omega_arg(omega, widths)
    h = np.empty((nout, L), np.float64)
    _load().orc_filter_gen_1d(ctypes.c_int64(L), ctypes.c_int(F), ctypes.c_int(int(include_t)),
                              ctypes.c_int(len(Ws)), warr, _ptr_array(Ws), _ptr_array(bs),
                              _dp(alpha), ctypes.c_int(ACT[act]), omp, ctypes.c_int(WINDOW[window]), _dp(h))
    return h


def filter_gen_3d_points(g, circular, F, Ws, bs, gamma, beta, alpha, idx, act="silu", omega=None,
                         window="exp") -> np.ndarray:
    """Kernel values at flat transform-grid indices idx: shape (len(idx), n_out)."""
    Ws, bs, widths, warr = _mlp_args(Ws, bs)
    alpha = _f64(alpha)
    idx = np.ascontiguousarray(np.asarray(idx, np.int64))
    out = np.empty((idx.size, widths[-1]), np.float64)
    gp = bp = None
    if gamma is not None:
        gamma = _f64(gamma); beta = _f64(beta)
        gp, bp = _dp(gamma), _dp(beta)
    om, omp = _omega_arg(omega, widths)
    _load().orc_filter_gen_3d_points(ctypes.c_int(g), ctypes.c_int(int(circular)), ctypes.c_int(F),
                                     ctypes.c_int(len(Ws)), warr, _ptr_array(Ws), _ptr_array(bs),
                                     gp, bp, _dp(alpha), ctypes.c_int(ACT[act]), omp, ctypes.c_int(WINDOW[window]),
                                     ctypes.c_int64(idx.size), _ip(idx), _dp(out))
    return out


def filter_gen_3d(g, circular, F, Ws, bs, gamma, beta, alpha) -> np.ndarray:
    """Whole kernel on the transform grid: shape (n_out, S, S, S)."""
    S = g if circular else 2 * g
    idx = np.arange(S ** 3, dtype=np.int64)
    pts = filter_gen_3d_points(g, circular, F, Ws, bs, gamma, beta, alpha, idx)
    return np.ascontiguousarray(pts.T.reshape(-1, S, S, S))


# --------------------------------------------------------------------------
# a3: filter spectrum (direct DFT)
# --------------------------------------------------------------------------

def dft_real_rows(h: np.ndarray, n: int) -> np.ndarray:
    """H[r, k] = sum_t h[r, t] e^{-2 pi i k t / n}, k = 0..n/2 (direct)."""
    h = _f64(h)
    rows, L = h.reshape(-1, h.shape[-1]).shape
    nb = n // 2 + 1
    re = np.empty((rows, nb)); im = np.empty((rows, nb))
    _load().orc_dft_real_rows(ctypes.c_int64(rows), ctypes.c_int64(L), ctypes.c_int64(n),
                              _dp(h), _dp(re), _dp(im))
    return (re + 1j * im).reshape(h.shape[:-1] + (nb,))


# --------------------------------------------------------------------------
# a4-a7: causal convolution and the gating chain (direct)
# --------------------------------------------------------------------------

def causal_conv(h, u, Dk: float = 0.0) -> np.ndarray:
    h = _f64(h); u = _f64(u)
    L = u.shape[0]
    assert h.shape == (L,)
    c = np.empty(L)
    _load().orc_causal_conv(ctypes.c_int64(L), _dp(h), _dp(u), ctypes.c_double(Dk), _dp(c))
    return c


def hyena_rows(v, xs, h, Dskip, rows=None, T=None) -> np.ndarray:
    """Order-(K+1) chain on selected rows (flat b*D+d), first T outputs.

    v, xs[k]: (B, D, L); h: (K, D, L); Dskip: (K, D) or None.
    Returns (len(rows), T)."""
    v = _f64(v)
    B, D, L = v.shape
    xs = [_f64(x) for x in xs]
    K = len(xs)
    h = _f64(h)
    assert h.shape == (K, D, L)
    if rows is None:
        rows = np.arange(B * D, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    T = L if T is None else int(T)
    y = np.empty((rows.size, T))
    dsk = None
    if Dskip is not None:
        Dskip = _f64(Dskip)
        dsk = _dp(Dskip)
    _load().orc_hyena_rows(ctypes.c_int(K), ctypes.c_int64(B), ctypes.c_int64(D), ctypes.c_int64(L),
                           ctypes.c_int64(T), _dp(v), _ptr_array(xs), _dp(h), dsk,
                           ctypes.c_int64(rows.size), _ip(rows), _dp(y))
    return y


def _causal_matrix(h: np.ndarray) -> np.ndarray:
    """T[t, s] = h[t - s] for t >= s, else 0: c = T z is the causal convolution."""
    L = h.shape[0]
    idx = np.arange(L)[:, None] - np.arange(L)[None, :]
    return np.where(idx >= 0, h[np.clip(idx, 0, L - 1)], 0.0)


def hyena_backward(v, xs, h, Dskip, dy):
    """Gradients of the order-N operator ([HN] 아키텍처 상세, step 3,
    differentiated), float64, by explicit matrices: with T_k the causal
    convolution matrix of h_k, c_k = T_k z_{k-1} + D_k z_{k-1}, so the
    adjoint is g_{k-1} = T_k^T e_k + D_k e_k with e_k = g_k x_k; dx_k =
    g_k c_k; dh_k[tau] = sum_b sum_t e_k[t] z_{k-1}[t - tau] (the matrix of
    z_{k-1} transposed times e_k); dD_k = sum_b e_k . z_{k-1}.

    v, xs[k], dy: (B, D, L); h: (K, D, L); Dskip: (K, D) or None.
    Returns (dv, [dx_k], dh (K, D, L), dD (K, D))."""
    v = np.asarray(v, np.float64)
    dy = np.asarray(dy, np.float64)
    xs = [np.asarray(x, np.float64) for x in xs]
    h = np.asarray(h, np.float64)
    K = h.shape[0]
    B, D, L = v.shape
    Dk = np.zeros((K, D)) if Dskip is None else np.asarray(Dskip, np.float64)
    dv = np.empty_like(v)
    dxs = [np.empty_like(v) for _ in range(K)]
    dh = np.zeros((K, D, L))
    dD = np.zeros((K, D))
    for d in range(D):
        T = [_causal_matrix(h[k, d]) for k in range(K)]
        for b in range(B):
            z = [v[b, d]]
            c = []
            for k in range(K):
                c.append(T[k] @ z[k] + Dk[k, d] * z[k])
                z.append(xs[k][b, d] * c[k])
            g = dy[b, d]
            for k in range(K - 1, -1, -1):
                dxs[k][b, d] = g * c[k]
                e = g * xs[k][b, d]
                dh[k, d] += _causal_matrix(z[k]).T @ e
                dD[k, d] += e @ z[k]
                g = T[k].T @ e + Dk[k, d] * e
            dv[b, d] = g
    return dv, dxs, dh, dD


def hyena_backward_samples(v, x1, h, Dk, dy, ts):
    """Order-2 gradients by their direct sums at chosen indices, float64:
    for each row (b, d) and s in ts
      dv[s] = sum_{t>=s} h[t-s] e[t] + D e[s],  e = dy x1,
      dx1[s] = dy[s] (sum_{u<=s} h[s-u] v[u] + D v[s]),
    and for each lag tau in ts dh[d, tau] = sum_b sum_{t>=tau} e[t] v[t-tau];
    dD[d] = sum_b e . v in full.  v, x1, dy: (B, D, L); h: (D, L); Dk: (D,)
    or None.  Returns (dv (B, D, n), dx1 (B, D, n), dh (D, n), dD (D,))."""
    v, x1, dy, h = (np.asarray(a, np.float64) for a in (v, x1, dy, h))
    ts = np.asarray(ts, np.int64)
    B, D, L = v.shape
    Dk = np.zeros(D) if Dk is None else np.asarray(Dk, np.float64)
    e = dy * x1
    dv = np.empty((B, D, ts.size))
    dx = np.empty((B, D, ts.size))
    dh = np.zeros((D, ts.size))
    for b in range(B):
        for d in range(D):
            for j, s in enumerate(ts):
                dv[b, d, j] = float(h[d, :L - s] @ e[b, d, s:]) + Dk[d] * e[b, d, s]
                dx[b, d, j] = dy[b, d, s] * (float(h[d, :s + 1][::-1] @ v[b, d, :s + 1]) + Dk[d] * v[b, d, s])
                dh[d, j] += float(e[b, d, s:] @ v[b, d, :L - s])
    dD = np.einsum("bdt,bdt->d", e, v)
    return dv, dx, dh, dD


def conv_gate_samples(h, u, x, Dk, ts) -> np.ndarray:
    """x[t] * (sum_{s<=t} h[t-s] u[s] + Dk u[t]) at the given t (one row)."""
    h = _f64(h); u = _f64(u)
    ts = np.ascontiguousarray(np.asarray(ts, np.int64))
    out = np.empty(ts.size)
    xp = None
    if x is not None:
        x = _f64(x)
        xp = _dp(x)
    _load().orc_conv_gate_samples(ctypes.c_int64(u.shape[0]), _dp(h), _dp(u), xp,
                                  ctypes.c_double(Dk), ctypes.c_int64(ts.size), _ip(ts), _dp(out))
    return out


# --------------------------------------------------------------------------
# a9: N-D convolution (direct, sampled voxels)
# --------------------------------------------------------------------------

def nd_conv_points(Kern, v, x1, Dk, pts, circular=False) -> np.ndarray:
    v = _f64(v)
    g = v.shape
    assert len(g) == 3
    Kern = _f64(Kern)
    S = g if circular else tuple(2 * a for a in g)
    assert Kern.shape == S, (Kern.shape, S)
    pts = np.ascontiguousarray(np.asarray(pts, np.int64))
    out = np.empty(pts.size)
    xp = None
    if x1 is not None:
        x1 = _f64(x1)
        xp = _dp(x1)
    garr = (ctypes.c_int * 3)(*g)
    _load().orc_nd_conv_points(garr, ctypes.c_int(int(circular)), _dp(Kern), _dp(v), xp,
                               ctypes.c_double(Dk), ctypes.c_int64(pts.size), _ip(pts), _dp(out))
    return out


# --------------------------------------------------------------------------
# a10: spectral gate (direct)
# --------------------------------------------------------------------------

def gate_kernel(g: np.ndarray) -> np.ndarray:
    """kappa = irFFT_n(g) by the direct inverse DFT; g has n/2+1 bins."""
    g = np.asarray(g, np.complex128)
    n = 2 * (g.shape[-1] - 1)
    re = _f64(g.real); im = _f64(g.imag)
    kap = np.empty(n)
    _load().orc_gate_kernel(ctypes.c_int64(n), _dp(re), _dp(im), _dp(kap))
    return kap


def circular_conv_samples(kappa, x1, x2, ts) -> np.ndarray:
    kappa = _f64(kappa); x1 = _f64(x1)
    ts = np.ascontiguousarray(np.asarray(ts, np.int64))
    out = np.empty(ts.size)
    xp = None
    if x2 is not None:
        x2 = _f64(x2)
        xp = _dp(x2)
    _load().orc_circular_conv_samples(ctypes.c_int64(kappa.shape[0]), _dp(kappa), _dp(x1), xp,
                                      ctypes.c_int64(ts.size), _ip(ts), _dp(out))
    return out


def prefix_gate_outputs(g, x1, x2, T: int) -> np.ndarray:
    """Streaming reading of the spectral gate ([SP] 토큰 믹서 구성과 생성 지원):
    output n < T is the full gated circular convolution of the sequence whose
    positions after n are zero, at position n.  g: n/2+1 bins; x1, x2:
    length-n rows (x2 may be None).  Returns (T,)."""
    kap = gate_kernel(g)
    x1 = _f64(x1)
    out = np.empty(T)
    for n in range(T):
        xp = x1.copy()
        xp[n + 1:] = 0.0
        out[n] = circular_conv_samples(kap, xp, None if x2 is None else _f64(x2), [n])[0]
    return out


def circular_conv_rows(kap, kidx, x1, x2) -> np.ndarray:
    """Rows x1 (R, n) convolved circularly with kap[kidx[r]], gated by x2."""
    kap = _f64(kap); x1 = _f64(x1)
    R, n = x1.shape
    kidx = np.ascontiguousarray(np.asarray(kidx, np.int64))
    y = np.empty((R, n))
    xp = None
    if x2 is not None:
        x2 = _f64(x2)
        xp = _dp(x2)
    _load().orc_circular_conv_rows(ctypes.c_int64(n), ctypes.c_int64(R), _dp(kap), _ip(kidx),
                                   _dp(x1), xp, _dp(y))
    return y


# --------------------------------------------------------------------------
# FFT-route references (numpy.fft as a library step, float64)
# --------------------------------------------------------------------------

def transform_len(L: int) -> int:
    """Smallest power of two >= 2L: zero-padding to it makes the FFT product a
    linear (not circular) convolution ([HN] fft_conv, [ND] 경계 처리)."""
    n = 1
    while n < 2 * L:
        n *= 2
    return n


def fft_spectrum(h: np.ndarray, n: int | None = None) -> np.ndarray:
    """rFFT of each zero-padded filter row: (..., n/2+1) complex128."""
    h = _f64(h)
    n = transform_len(h.shape[-1]) if n is None else n
    return np.fft.rfft(h, n=n, axis=-1)


def fft_hyena_rows(v, xs, h, Dskip, rows=None) -> np.ndarray:
    """The order-(K+1) chain of [HN] step 3 with each h_k * z by the padded FFT.

    Same layouts as hyena_rows; returns (len(rows), L)."""
    v = _f64(v)
    B, D, L = v.shape
    K = len(xs)
    n = transform_len(L)
    if rows is None:
        rows = np.arange(B * D)
    rows = np.asarray(rows, np.int64)
    d = rows % D
    out = np.empty((rows.size, L))
    chunk = max(1, (1 << 24) // n)
    for s in range(0, rows.size, chunk):
        r = rows[s:s + chunk]
        dd = d[s:s + chunk]
        z = v.reshape(B * D, L)[r]
        for k in range(K):
            Hk = np.fft.rfft(_f64(h[k])[dd], n=n, axis=-1)
            c = np.fft.irfft(np.fft.rfft(z, n=n, axis=-1) * Hk, n=n, axis=-1)[:, :L]
            if Dskip is not None:
                c = c + _f64(Dskip)[k][dd][:, None] * z
            z = _f64(xs[k]).reshape(B * D, L)[r] * c
        out[s:s + chunk] = z
    return out


def fft_nd_conv(Kern, v, x1, Dk=0.0, circular=False) -> np.ndarray:
    """[ND] N-D convolution of one slab through the 3-D FFT, cropped to the grid."""
    v = _f64(v)
    g = v.shape
    S = g if circular else tuple(2 * a for a in g)
    Hk = np.fft.rfftn(_f64(Kern), s=S, axes=(0, 1, 2))
    c = np.fft.irfftn(np.fft.rfftn(v, s=S, axes=(0, 1, 2)) * Hk, s=S, axes=(0, 1, 2))[: g[0], : g[1], : g[2]]
    c = c + Dk * v
    return c if x1 is None else _f64(x1) * c


def fft_spectral_gate_rows(g_rows, x1, x2) -> np.ndarray:
    """[SP] y = x2 * irFFT(g * rFFT(x1)) with the imaginary part of the product
    dropped at the DC and Nyquist bins (numpy's irfft does exactly that)."""
    x1 = _f64(x1)
    n = x1.shape[-1]
    y = np.fft.irfft(np.fft.rfft(x1, axis=-1) * np.asarray(g_rows, np.complex128), n=n, axis=-1)
    return y if x2 is None else _f64(x2) * y


# --------------------------------------------------------------------------
# naive float64 CPU FFT route (fft_reference.c): the baseline program timed
# beside the direct oracle
# --------------------------------------------------------------------------

def fftref_fft(x, inverse: bool = False) -> np.ndarray:
    """Unnormalised DFT of a complex vector (length a power of two) by the
    naive radix-2 FFT: X[k] = sum_j x[j] exp(-+2 pi i jk/n)."""
    x = np.asarray(x, np.complex128)
    re = np.ascontiguousarray(x.real)
    im = np.ascontiguousarray(x.imag)
    _load().fref_fft(ctypes.c_int64(x.size), _dp(re), _dp(im), ctypes.c_int(1 if inverse else 0))
    return re + 1j * im


def fftref_hyena_rows(v, xs, h, Dskip, rows=None) -> np.ndarray:
    """The order-(K+1) chain of hyena_rows through the naive FFT route
    (zero-padded to transform_len(L), filter transform per row)."""
    v = _f64(v)
    B, D, L = v.shape
    xs = [_f64(x) for x in xs]
    K = len(xs)
    h = _f64(h)
    assert h.shape == (K, D, L)
    if rows is None:
        rows = np.arange(B * D, dtype=np.int64)
    rows = np.ascontiguousarray(np.asarray(rows, np.int64))
    y = np.empty((rows.size, L))
    dsk = None
    if Dskip is not None:
        Dskip = _f64(Dskip)
        dsk = _dp(Dskip)
    _load().fref_hyena_rows(ctypes.c_int(K), ctypes.c_int64(D), ctypes.c_int64(L),
                            ctypes.c_int64(transform_len(L)), _dp(v), _ptr_array(xs), _dp(h), dsk,
                            ctypes.c_int64(rows.size), _ip(rows), _dp(y))
    return y


def fftref_gate_rows(g, gidx, x1, x2) -> np.ndarray:
    """Spectral gate rows through the naive FFT route.  g: (nk, n/2+1)
    complex; gidx: the g row of each x1 row; x1, x2: (nrows, n) (x2 may be None)."""
    x1 = _f64(x1)
    nrows, n = x1.shape
    g = np.asarray(g, np.complex128)
    gre, gim = np.ascontiguousarray(g.real), np.ascontiguousarray(g.imag)
    gidx = np.ascontiguousarray(np.asarray(gidx, np.int64))
    y = np.empty((nrows, n))
    x2keep = _f64(x2) if x2 is not None else None
    x2p = _dp(x2keep) if x2keep is not None else None
    _load().fref_gate_rows(ctypes.c_int64(n), ctypes.c_int64(nrows), _dp(gre), _dp(gim), _ip(gidx),
                           _dp(x1), x2p, _dp(y))
    return y


def fftref_nd_conv(Kern, kidx, v, x1, circular: bool = False) -> np.ndarray:
    """Gated N-D convolution of slabs v (nslab, g0, g1, g2) through the naive
    FFT route; Kern (nk, S0, S1, S2) on the transform grid, slab s using
    Kern[kidx[s]]; x1 like v or None.  No skip term."""
    v = _f64(v)
    nslab = v.shape[0]
    g = (ctypes.c_int * 3)(*v.shape[1:])
    Kern = _f64(Kern)
    kidx = np.ascontiguousarray(np.asarray(kidx, np.int64))
    y = np.empty_like(v)
    x1keep = _f64(x1) if x1 is not None else None
    _load().fref_nd_conv(g, ctypes.c_int(1 if circular else 0), ctypes.c_int64(nslab), _dp(Kern), _ip(kidx),
                         _dp(v), _dp(x1keep) if x1keep is not None else None, _dp(y))
    return y
