/*
 * hyena_oracle.c -- plain, slow, float64 reference for the Hyena hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or constant
 * with the CUDA library: every formula here is written out from its
 * definition on the pages, in float64, with no FFT, no blocking and no fusion.
 *
 * Pages cited (by title and section):
 *   [HN]  "Hyena: 암묵적 장거리 컨볼루션으로 어텐션을 완전 대체한 서브-이차 모델"
 *         -- 아키텍처 상세 (step 2 filter equation h(t)=FFN(pos_enc(t))·w(t),
 *         w(t)=e^{-αt}; step 3 gating equation), and its ImplicitFilter /
 *         hyena_operator code sketch.
 *   [ES]  "4. Hyena 상세" -- 어떻게 동작하나요? (filter generator with
 *         sinusoidal features and exponential decay; FFT convolution with a
 *         filter as long as the sequence).
 *   [ND]  "Native Multi-Dimensional Subquadratic Operators via Input Dependent
 *         Long Convolutions" -- 방법론: HyenaND (네이티브 ND 합성곱, 경계 처리:
 *         circular or non-circular by zero-padding each axis to double).
 *   [SP]  "FFT의 반격: Self-Attention의 효율적 대안" -- 토큰 믹서 구성과 생성
 *         지원 (real FFT, spectral gate on n/2+1 bins, inverse FFT).
 *
 * Every function is exact up to float64 rounding order.  All sums run in
 * increasing index order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_PI 3.14159265358979323846264338327950288

/* ------------------------------------------------------------------------ */
/* a1: sinusoidal positional encoding                                        */
/* ------------------------------------------------------------------------ */

/* [HN] step 2: the filter is a small FFN of a positional encoding of t; the
 * ImplicitFilter sketch uses a sine/cosine basis.  [ES] names "sinusoidal
 * features".  Frequencies are not given; the reading used here is harmonics
 * j = 1..F of the normalised position t/L:
 *   PE(t) = [t/L (optional), cos(2π j t/L) for j=1..F, sin(2π j t/L) for j=1..F]
 * The angle is reduced exactly in integers, (j·t mod L)/L, before cos/sin.
 * out is row-major (L x width), width = include_t + 2F. */
void orc_pe1d(int64_t L, int F, int include_t, double *out)
{
    const int w = include_t + 2 * F;
    for (int64_t t = 0; t < L; ++t) {
        double *row = out + t * w;
        int c = 0;
        if (include_t) row[c++] = (double)t / (double)L;
        for (int j = 1; j <= F; ++j) {
            int64_t r = ((int64_t)j * t) % L;
            row[c + j - 1] = cos(2.0 * ORC_PI * (double)r / (double)L);
            row[c + F + j - 1] = sin(2.0 * ORC_PI * (double)r / (double)L);
        }
    }
}

/* 3-D encoding of a signed lattice offset r = (rx, ry, rz), each axis scaled
 * by the unpadded edge g: per axis a, features cos(π j r_a/g), sin(π j r_a/g)
 * for j = 1..F (axis-major: x cos.., x sin.., y cos.., ...).  [ND] builds the
 * kernel from a coordinate MLP on the grid; the pages give no frequencies,
 * this is the reading taken (one half-period over the unit coordinate). */
static void orc_pe3d_point(int g, int F, const int r[3], double *out)
{
    for (int a = 0; a < 3; ++a) {
        int64_t twog = 2 * (int64_t)g;
        for (int j = 1; j <= F; ++j) {
            /* angle π j r/g = 2π (j r mod 2g)/(2g), reduced exactly */
            int64_t m = ((int64_t)j * r[a]) % twog;
            if (m < 0) m += twog;
            double ang = 2.0 * ORC_PI * (double)m / (double)twog;
            out[a * 2 * F + j - 1] = cos(ang);
            out[a * 2 * F + F + j - 1] = sin(ang);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a2: the filter MLP and the decay window                                   */
/* ------------------------------------------------------------------------ */

static double orc_silu(double a) { return a / (1.0 + exp(-a)); }

/* One position through the MLP.  Layer l maps widths[l] -> widths[l+1]:
 * y = W_l x + b_l with W_l row-major (out x in).  Hidden layers (all but the
 * last) optionally get FiLM on the first hidden layer, y <- (1+γ)⊙y + β
 * ([ND] FiLM conditioning of the kernel MLP), then SiLU ([HN] sketch).  */
/* Hidden activation: 0 SiLU, 1 identity, 2 sine sin(ω x) (SIREN, [ND]
 * 방법론: 좌표 기반 SIREN MLP; ω per hidden unit, 1 when omega is NULL). */
static double orc_act(int act, double s, double w)
{
    if (act == 1) return s;
    if (act == 2) return sin(w * s);
    return orc_silu(s);
}

static void orc_mlp_point(int nl, const int *widths, const double *const *W,
                          const double *const *b, const double *film_gamma,
                          const double *film_beta, int act, const double *omega,
                          const double *x, double *out, double *scratch_a, double *scratch_b)
{
    const double *cur = x;
    int64_t woff = 0;   /* offset of this hidden layer's frequencies in omega */
    for (int l = 0; l < nl; ++l) {
        int win = widths[l], wout = widths[l + 1];
        double *dst = (l == nl - 1) ? out : ((l & 1) ? scratch_b : scratch_a);
        for (int o = 0; o < wout; ++o) {
            double s = b[l][o];
            const double *wr = W[l] + (int64_t)o * win;
            for (int i = 0; i < win; ++i) s += wr[i] * cur[i];
            if (l < nl - 1) {
                if (l == 0 && film_gamma) s = (1.0 + film_gamma[o]) * s + film_beta[o];
                s = orc_act(act, s, omega ? omega[woff + o] : 1.0);
            }
            dst[o] = s;
        }
        if (l < nl - 1) woff += wout;
        cur = dst;
    }
}

/* Window on the normalised distance n (t/L or |r|/g): 0 exponential
 * exp(-α n) ([HN] w(t) = e^{-αt}), 1 Gaussian exp(-α n²) ([ND] 커널 합성:
 * 학습 가능한 가우시안 윈도우, α = 1/(2σ²)). */
static double orc_window(int window, double alpha, double n)
{
    return window == 1 ? exp(-alpha * n * n) : exp(-alpha * n);
}

static int orc_max_width(int nl, const int *widths)
{
    int m = 0;
    for (int l = 0; l <= nl; ++l) if (widths[l] > m) m = widths[l];
    return m;
}

/* [HN] step 2 and the ImplicitFilter sketch: h(t) = FFN(PE(t)) · w(t).  The
 * decay is one rate per output column, α_o ≥ 0, on normalised time:
 *   h[o, t] = MLP(PE(t))[o] · exp(-α_o · t / L),   o < n_out, t < L.
 * h is row-major (n_out x L).  n_out = K·D for an operator with K filters. */
void orc_filter_gen_1d(int64_t L, int F, int include_t, int nl, const int *widths,
                       const double *const *W, const double *const *b,
                       const double *alpha, int act, const double *omega, int window, double *h)
{
    const int win = widths[0];
    const int nout = widths[nl];
    const int mw = orc_max_width(nl, widths);
    #pragma omp parallel
    {
        double *pe = (double *)malloc(sizeof(double) * (size_t)win);
        double *sa = (double *)malloc(sizeof(double) * (size_t)mw);
        double *sb = (double *)malloc(sizeof(double) * (size_t)mw);
        double *o = (double *)malloc(sizeof(double) * (size_t)nout);
        #pragma omp for schedule(static)
        for (int64_t t = 0; t < L; ++t) {
            int c = 0;
            if (include_t) pe[c++] = (double)t / (double)L;
            for (int j = 1; j <= F; ++j) {
                int64_t r = ((int64_t)j * t) % L;
                pe[c + j - 1] = cos(2.0 * ORC_PI * (double)r / (double)L);
                pe[c + F + j - 1] = sin(2.0 * ORC_PI * (double)r / (double)L);
            }
            orc_mlp_point(nl, widths, W, b, NULL, NULL, act, omega, pe, o, sa, sb);
            double tn = (double)t / (double)L;
            for (int k = 0; k < nout; ++k) h[(int64_t)k * L + t] = o[k] * orc_window(window, alpha[k], tn);
        }
        free(pe); free(sa); free(sb); free(o);
    }
}

/* Signed offset of grid index i on a transform axis of size S:
 * i < S/2 -> i, else i - S. */
static int orc_signed_offset(int64_t i, int64_t S) { return (int)(i < S / 2 ? i : i - S); }

/* [ND] native N-D kernel K(r) from a coordinate MLP with FiLM conditioning and
 * a decay envelope (reading: exp(-α‖r‖/g) in place of the learnable window).
 * The kernel lives on the transform grid of edge S (S = 2g non-circular,
 * S = g circular) with wrap indexing of signed offsets.  In the non-circular
 * case only |r_a| ≤ g-1 is in the support; index S/2 (offset -g) is zero.
 * Evaluates npts grid points given by flat index p = (ix·S + iy)·S + iz;
 * out is (npts x n_out).  gamma/beta: FiLM of the first hidden layer for
 * this sample (NULL for none). */
void orc_filter_gen_3d_points(int g, int circular, int F, int nl, const int *widths,
                              const double *const *W, const double *const *b,
                              const double *film_gamma, const double *film_beta,
                              const double *alpha, int act, const double *omega, int window,
                              int64_t npts, const int64_t *idx, double *out)
{
    const int64_t S = circular ? (int64_t)g : 2 * (int64_t)g;
    const int nout = widths[nl];
    const int mw = orc_max_width(nl, widths);
    #pragma omp parallel
    {
        double *pe = (double *)malloc(sizeof(double) * (size_t)(6 * F));
        double *sa = (double *)malloc(sizeof(double) * (size_t)mw);
        double *sb = (double *)malloc(sizeof(double) * (size_t)mw);
        double *o = (double *)malloc(sizeof(double) * (size_t)nout);
        #pragma omp for schedule(static)
        for (int64_t q = 0; q < npts; ++q) {
            int64_t p = idx[q];
            int64_t ix = p / (S * S), iy = (p / S) % S, iz = p % S;
            int r[3] = {orc_signed_offset(ix, S), orc_signed_offset(iy, S), orc_signed_offset(iz, S)};
            int inside = 1;
            if (!circular)
                for (int a = 0; a < 3; ++a) if (r[a] <= -g || r[a] >= g) inside = 0;
            double *row = out + q * nout;
            if (!inside) { for (int k = 0; k < nout; ++k) row[k] = 0.0; continue; }
            orc_pe3d_point(g, F, r, pe);
            orc_mlp_point(nl, widths, W, b, film_gamma, film_beta, act, omega, pe, o, sa, sb);
            double rn = sqrt((double)r[0] * r[0] + (double)r[1] * r[1] + (double)r[2] * r[2]) / (double)g;
            for (int k = 0; k < nout; ++k) row[k] = o[k] * orc_window(window, alpha[k], rn);
        }
        free(pe); free(sa); free(sb); free(o);
    }
}

/* ------------------------------------------------------------------------ */
/* a3: filter spectrum, by the direct DFT                                    */
/* ------------------------------------------------------------------------ */

/* The spectrum of the zero-padded filter that the FFT convolution multiplies
 * by ([HN] fft_conv, [ES] "FFT → 원소별 곱 → 역 FFT"):
 *   H[k] = Σ_{t<L} h[t] e^{-2πi k t / n},  k = 0..n/2,  n = transform length.
 * Direct O(L·n) sum; the angle (k·t mod n) is reduced exactly. */
void orc_dft_real_rows(int64_t nrows, int64_t L, int64_t n, const double *h,
                       double *Hre, double *Him)
{
    const int64_t nb = n / 2 + 1;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < nrows; ++r) {
        const double *hr = h + r * L;
        for (int64_t k = 0; k < nb; ++k) {
            double sr = 0.0, si = 0.0;
            for (int64_t t = 0; t < L; ++t) {
                int64_t m = (k * t) % n;
                double ang = -2.0 * ORC_PI * (double)m / (double)n;
                sr += hr[t] * cos(ang);
                si += hr[t] * sin(ang);
            }
            Hre[r * nb + k] = sr;
            Him[r * nb + k] = si;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* a4-a7: causal long convolution, skip term and the gating chain            */
/* ------------------------------------------------------------------------ */

/* Causal convolution with a filter as long as the sequence ([ES]: "커널 크기를
 * 시퀀스 전체 길이 N 만큼"), plus the D·u skip term:
 *   c[t] = Σ_{s=0}^{t} h[t-s] u[s] + Dk·u[t],  t = 0..T-1  (T ≤ L).
 * Direct O(T²); zero-padding to 2L in the FFT route makes it equal to this. */
static void orc_causal_conv_prefix(int64_t T, const double *h, const double *u,
                                   double Dk, double *c)
{
    for (int64_t t = 0; t < T; ++t) {
        double s = 0.0;
        for (int64_t q = 0; q <= t; ++q) s += h[t - q] * u[q];
        c[t] = s + Dk * u[t];
    }
}

void orc_causal_conv(int64_t L, const double *h, const double *u, double Dk, double *c)
{
    orc_causal_conv_prefix(L, h, u, Dk, c);
}

/* The order-N recurrence of [HN] step 3 and the hyena_operator sketch:
 *   z_0 = v;  z_k = x_k ⊙ (h_k * z_{k-1} + D_k ⊙ z_{k-1}),  k = 1..K;  y = z_K.
 * Layouts: v, x[k], y are (B, D, L) row-major; h is (K, D, L) shared across
 * the batch; Dskip is (K, D) or NULL (no skip).  Only the first T outputs of
 * each requested row are computed (T = L for whole rows): the chain is causal,
 * so a prefix depends on input prefixes only.  rows[] lists flat row indices
 * b·D + d; y is (nrows x T). */
void orc_hyena_rows(int K, int64_t B, int64_t D, int64_t L, int64_t T,
                    const double *v, const double *const *x, const double *h,
                    const double *Dskip, int64_t nrows, const int64_t *rows,
                    double *y)
{
    (void)B;
    #pragma omp parallel
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)T);
        double *c = (double *)malloc(sizeof(double) * (size_t)T);
        #pragma omp for schedule(dynamic)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t row = rows[i];
            int64_t d = row % D;
            memcpy(z, v + row * L, sizeof(double) * (size_t)T);
            for (int k = 0; k < K; ++k) {
                const double *hk = h + ((int64_t)k * D + d) * L;
                double Dk = Dskip ? Dskip[(int64_t)k * D + d] : 0.0;
                orc_causal_conv_prefix(T, hk, z, Dk, c);
                const double *xk = x[k] + row * L;
                for (int64_t t = 0; t < T; ++t) z[t] = xk[t] * c[t];
            }
            memcpy(y + i * T, z, sizeof(double) * (size_t)T);
        }
        free(z); free(c);
    }
}

/* Single samples of one order of the chain, for rows too long for the O(T²)
 * prefix:  out[i] = x[t_i] · (Σ_{s≤t_i} h[t_i-s] u[s] + Dk·u[t_i]).
 * u, h, x are one row each (length L). */
void orc_conv_gate_samples(int64_t L, const double *h, const double *u, const double *x,
                           double Dk, int64_t ns, const int64_t *ts, double *out)
{
    (void)L;
    #pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < ns; ++i) {
        int64_t t = ts[i];
        double s = 0.0;
        for (int64_t q = 0; q <= t; ++q) s += h[t - q] * u[q];
        s += Dk * u[t];
        out[i] = x ? x[t] * s : s;
    }
}

/* ------------------------------------------------------------------------ */
/* a9: N-D global convolution with gating (HyenaND)                          */
/* ------------------------------------------------------------------------ */

/* [ND] 네이티브 ND 합성곱 and 경계 처리.  On a g0 x g1 x g2 grid, for output
 * voxel p:
 *   non-circular:  c[p] = Σ_{q in grid} K[(p - q) mod S] v[q],  S = 2g per axis
 *                  (zero-padding each axis to double: a linear convolution)
 *   circular:      c[p] = Σ_q K[(p - q) mod g] v[q]  (periodic systems)
 *   y[p] = x1[p] · (c[p] + Dk · v[p])
 * K is one kernel on the transform grid (S0 x S1 x S2), v/x1 one slab
 * (g0 x g1 x g2).  Evaluates ns voxels given by flat index (i·g1 + j)·g2 + l. */
void orc_nd_conv_points(const int *g, int circular, const double *Kern,
                        const double *v, const double *x1, double Dk,
                        int64_t ns, const int64_t *pts, double *out)
{
    int64_t S[3];
    for (int a = 0; a < 3; ++a) S[a] = circular ? g[a] : 2 * (int64_t)g[a];
    #pragma omp parallel for schedule(dynamic)
    for (int64_t n = 0; n < ns; ++n) {
        int64_t p = pts[n];
        int64_t pi = p / ((int64_t)g[1] * g[2]), pj = (p / g[2]) % g[1], pl = p % g[2];
        double s = 0.0;
        for (int64_t i = 0; i < g[0]; ++i) {
            int64_t di = ((pi - i) % S[0] + S[0]) % S[0];
            for (int64_t j = 0; j < g[1]; ++j) {
                int64_t dj = ((pj - j) % S[1] + S[1]) % S[1];
                const double *vr = v + (i * g[1] + j) * g[2];
                const double *kr = Kern + (di * S[1] + dj) * S[2];
                for (int64_t l = 0; l < g[2]; ++l) {
                    int64_t dl = ((pl - l) % S[2] + S[2]) % S[2];
                    s += kr[dl] * vr[l];
                }
            }
        }
        s += Dk * v[p];
        out[n] = x1 ? x1[p] * s : s;
    }
}

/* ------------------------------------------------------------------------ */
/* a10: spectral gating token mixer (SPECTRE-style), circular                 */
/* ------------------------------------------------------------------------ */

/* [SP] real FFT -> diagonal gate on the n/2+1 bins -> inverse FFT.  The gate
 * g[0..n/2] acts on a real signal, so the mixing is a circular convolution
 * with the real kernel κ = irFFT_n(g):
 *   κ[s] = (1/n) Σ_{k=0}^{n-1} G[k] e^{+2πi k s/n},
 *   G[k] = g[k] (k ≤ n/2), conj(g[n-k]) (k > n/2), with the imaginary part of
 *   g dropped at k = 0 and k = n/2 (the inverse real transform keeps only the
 *   real part there).
 * Direct inverse DFT, O(n²). */
void orc_gate_kernel(int64_t n, const double *gre, const double *gim, double *kappa)
{
    #pragma omp parallel for schedule(static)
    for (int64_t s = 0; s < n; ++s) {
        double acc = 0.0;
        for (int64_t k = 0; k < n; ++k) {
            double Gr, Gi;
            if (k == 0 || k == n / 2) { Gr = gre[k]; Gi = 0.0; }
            else if (k < n / 2) { Gr = gre[k]; Gi = gim[k]; }
            else { Gr = gre[n - k]; Gi = -gim[n - k]; }
            int64_t m = (k * s) % n;
            double ang = 2.0 * ORC_PI * (double)m / (double)n;
            /* Re(G e^{iθ}) -- the imaginary parts cancel over the Hermitian pair */
            acc += Gr * cos(ang) - Gi * sin(ang);
        }
        kappa[s] = acc / (double)n;
    }
}

/* y[t] = x2[t] · Σ_{s<n} κ[s] x1[(t - s) mod n]  (circular; x2 NULL = no gate).
 * Evaluates ns samples of one row. */
void orc_circular_conv_samples(int64_t n, const double *kappa, const double *x1,
                               const double *x2, int64_t ns, const int64_t *ts,
                               double *out)
{
    #pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < ns; ++i) {
        int64_t t = ts[i];
        double s = 0.0;
        for (int64_t q = 0; q < n; ++q) {
            int64_t j = ((t - q) % n + n) % n;
            s += kappa[q] * x1[j];
        }
        out[i] = x2 ? x2[t] * s : s;
    }
}

/* Whole rows of the circular convolution above: rows x1 (nrows x n), each
 * using kappa row kidx[r] of kap (nk x n), gated by x2 (or not). */
void orc_circular_conv_rows(int64_t n, int64_t nrows, const double *kap,
                            const int64_t *kidx, const double *x1, const double *x2,
                            double *y)
{
    #pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < nrows; ++r) {
        const double *kr = kap + kidx[r] * n;
        const double *xr = x1 + r * n;
        for (int64_t t = 0; t < n; ++t) {
            double s = 0.0;
            for (int64_t q = 0; q < n; ++q) {
                int64_t j = t - q;
                if (j < 0) j += n;
                s += kr[q] * xr[j];
            }
            y[r * n + t] = x2 ? x2[r * n + t] * s : s;
        }
    }
}
