/*
 * fft_reference.c -- a naive float64 CPU FFT route for the same quantities
 * as hyena_oracle.c: the baseline program that a CPU user of the method
 * would write first, timed beside the direct oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or
 * call this file; only the test-suite, the smoke check and the CPU-baseline
 * legs of the benchmark use it.  It shares no code, header, table or
 * constant with the CUDA library.  It is a reference, not the oracle: the
 * tests pin it to the direct definitions in hyena_oracle.c.
 *
 * The route is the one the pages describe for the long convolution
 * ([HN] "Hyena: 암묵적 장거리 컨볼루션으로 어텐션을 완전 대체한 서브-이차
 * 모델", fft_conv in the code sketch; [ES] "4. Hyena 상세", 어떻게
 * 동작하나요?: FFT, pointwise product, inverse FFT; [ND] "Native
 * Multi-Dimensional Subquadratic Operators via Input Dependent Long
 * Convolutions", 경계 처리: zero-pad each axis to double; [SP] "FFT의 반격:
 * Self-Attention의 효율적 대안", 토큰 믹서 구성과 생성 지원: real FFT, gate,
 * inverse FFT), written the plain way:
 *   - one iterative radix-2 complex FFT (bit-reversal permutation, then
 *     log2 n butterfly passes; each pass's twiddles from cos/sin of the
 *     exactly reduced angle), float64 throughout;
 *   - real signals go in as complex rows with a zero imaginary part (no
 *     real-to-complex packing), and the filter's transform is recomputed for
 *     every row, as the pages' sketch does inside fft_conv;
 *   - N-D transforms are 1-D transforms along each axis in turn.
 * OpenMP runs independent rows (or slabs) in parallel.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define FREF_PI 3.14159265358979323846264338327950288

/* In-place unnormalised DFT of length n (a power of two):
 *   X[k] = Σ_j x[j] e^{s·2πi jk/n},  s = -1 (forward) or +1 (inverse). */
void fref_fft(int64_t n, double *re, double *im, int inverse)
{
    /* bit-reversal permutation */
    for (int64_t i = 1, j = 0; i < n; ++i) {
        int64_t bit = n >> 1;
        for (; j & bit; bit >>= 1) j ^= bit;
        j ^= bit;
        if (i < j) {
            double t = re[i]; re[i] = re[j]; re[j] = t;
            t = im[i]; im[i] = im[j]; im[j] = t;
        }
    }
    const double sgn = inverse ? 1.0 : -1.0;
    for (int64_t len = 2; len <= n; len <<= 1) {
        const int64_t half = len >> 1;
        for (int64_t j = 0; j < half; ++j) {
            /* W_len^j = e^{s 2πi j/len}; j < len/2 needs no reduction */
            const double ang = sgn * 2.0 * FREF_PI * (double)j / (double)len;
            const double wr = cos(ang), wi = sin(ang);
            for (int64_t i = j; i < n; i += len) {
                const int64_t k = i + half;
                const double tr = re[k] * wr - im[k] * wi;
                const double ti = re[k] * wi + im[k] * wr;
                re[k] = re[i] - tr; im[k] = im[i] - ti;
                re[i] += tr; im[i] += ti;
            }
        }
    }
}

/* The order-(K+1) recurrence z_k = x_k ⊙ (h_k * z_{k-1} + D_k z_{k-1}) with
 * every causal convolution computed by the zero-padded FFT of length n
 * (a power of two >= 2L), then truncated to L.  Layouts as orc_hyena_rows:
 * v, x[k] (B, D, L); h (K, D, L); Dskip (K, D) or NULL; y (nrows, L). */
void fref_hyena_rows(int K, int64_t D, int64_t L, int64_t n, const double *v,
                     const double *const *x, const double *h, const double *Dskip,
                     int64_t nrows, const int64_t *rows, double *y)
{
    #pragma omp parallel
    {
        double *zr = (double *)malloc(sizeof(double) * (size_t)n);
        double *zi = (double *)malloc(sizeof(double) * (size_t)n);
        double *hr = (double *)malloc(sizeof(double) * (size_t)n);
        double *hi = (double *)malloc(sizeof(double) * (size_t)n);
        double *z = (double *)malloc(sizeof(double) * (size_t)L);
        #pragma omp for schedule(dynamic)
        for (int64_t i = 0; i < nrows; ++i) {
            const int64_t row = rows[i], d = row % D;
            memcpy(z, v + row * L, sizeof(double) * (size_t)L);
            for (int k = 0; k < K; ++k) {
                const double *hk = h + ((int64_t)k * D + d) * L;
                for (int64_t t = 0; t < n; ++t) {
                    zr[t] = t < L ? z[t] : 0.0;
                    hr[t] = t < L ? hk[t] : 0.0;
                    zi[t] = 0.0;
                    hi[t] = 0.0;
                }
                fref_fft(n, zr, zi, 0);
                fref_fft(n, hr, hi, 0);
                for (int64_t t = 0; t < n; ++t) {
                    const double a = zr[t] * hr[t] - zi[t] * hi[t];
                    const double b = zr[t] * hi[t] + zi[t] * hr[t];
                    zr[t] = a;
                    zi[t] = b;
                }
                fref_fft(n, zr, zi, 1);
                const double Dk = Dskip ? Dskip[(int64_t)k * D + d] : 0.0;
                const double *xk = x[k] + row * L;
                for (int64_t t = 0; t < L; ++t) z[t] = xk[t] * (zr[t] / (double)n + Dk * z[t]);
            }
            memcpy(y + i * L, z, sizeof(double) * (size_t)L);
        }
        free(zr); free(zi); free(hr); free(hi); free(z);
    }
}

/* The spectral gate on whole rows (circular, length n = L):
 *   y = x2 ⊙ irFFT(g ⊙ rFFT(x1)),
 * as a full complex transform: bins k > n/2 take conj(g[n-k]) and the
 * imaginary part of g is dropped at k = 0 and n/2, which is what the
 * inverse of a real transform does.  g rows are (n/2 + 1) complex, row r uses
 * g row gidx[r]; x2 may be NULL. */
void fref_gate_rows(int64_t n, int64_t nrows, const double *gre, const double *gim,
                    const int64_t *gidx, const double *x1, const double *x2, double *y)
{
    const int64_t nb = n / 2 + 1;
    #pragma omp parallel
    {
        double *re = (double *)malloc(sizeof(double) * (size_t)n);
        double *im = (double *)malloc(sizeof(double) * (size_t)n);
        #pragma omp for schedule(dynamic)
        for (int64_t r = 0; r < nrows; ++r) {
            const double *gr = gre + gidx[r] * nb, *gi = gim + gidx[r] * nb;
            for (int64_t t = 0; t < n; ++t) { re[t] = x1[r * n + t]; im[t] = 0.0; }
            fref_fft(n, re, im, 0);
            for (int64_t k = 0; k < n; ++k) {
                double Gr, Gi;
                if (k == 0 || k == n / 2) { Gr = gr[k]; Gi = 0.0; }
                else if (k < n / 2) { Gr = gr[k]; Gi = gi[k]; }
                else { Gr = gr[n - k]; Gi = -gi[n - k]; }
                const double a = re[k] * Gr - im[k] * Gi;
                const double b = re[k] * Gi + im[k] * Gr;
                re[k] = a;
                im[k] = b;
            }
            fref_fft(n, re, im, 1);
            for (int64_t t = 0; t < n; ++t) {
                const double c = re[t] / (double)n;
                y[r * n + t] = x2 ? x2[r * n + t] * c : c;
            }
        }
        free(re); free(im);
    }
}

/* 3-D transform of an S0 x S1 x S2 complex grid (row-major), one axis at a
 * time through a gathered line buffer. */
static void fref_fft3(const int64_t S[3], double *re, double *im, int inverse,
                      double *lr, double *li)
{
    const int64_t stride[3] = {S[1] * S[2], S[2], 1};
    for (int a = 0; a < 3; ++a) {
        const int b = a == 0 ? 1 : 0, c = a == 2 ? 1 : 2;
        for (int64_t ib = 0; ib < S[b]; ++ib)
            for (int64_t ic = 0; ic < S[c]; ++ic) {
                const int64_t base = ib * stride[b] + ic * stride[c];
                for (int64_t j = 0; j < S[a]; ++j) {
                    lr[j] = re[base + j * stride[a]];
                    li[j] = im[base + j * stride[a]];
                }
                fref_fft(S[a], lr, li, inverse);
                for (int64_t j = 0; j < S[a]; ++j) {
                    re[base + j * stride[a]] = lr[j];
                    im[base + j * stride[a]] = li[j];
                }
            }
    }
}

/* The gated N-D convolution of nslab slabs (b, d), without a skip term:
 *   y = x1 ⊙ crop_g(iFFT3(FFT3(pad_S v) ⊙ FFT3(K)) / (S0 S1 S2)),
 * S = 2g per axis (linear, zero-padded) or g (circular).  v, x1, y are
 * (nslab, g0, g1, g2); Kern is (nk, S0, S1, S2) on the transform grid, slab
 * s using kernel kidx[s]; x1 may be NULL. */
void fref_nd_conv(const int *g, int circular, int64_t nslab, const double *Kern,
                  const int64_t *kidx, const double *v, const double *x1, double *y)
{
    int64_t S[3];
    for (int a = 0; a < 3; ++a) S[a] = circular ? g[a] : 2 * (int64_t)g[a];
    const int64_t nS = S[0] * S[1] * S[2];
    const int64_t ng = (int64_t)g[0] * g[1] * g[2];
    int64_t smax = S[0] > S[1] ? S[0] : S[1];
    if (S[2] > smax) smax = S[2];
    #pragma omp parallel
    {
        double *vr = (double *)malloc(sizeof(double) * (size_t)nS);
        double *vi = (double *)malloc(sizeof(double) * (size_t)nS);
        double *kr = (double *)malloc(sizeof(double) * (size_t)nS);
        double *ki = (double *)malloc(sizeof(double) * (size_t)nS);
        double *lr = (double *)malloc(sizeof(double) * (size_t)smax);
        double *li = (double *)malloc(sizeof(double) * (size_t)smax);
        #pragma omp for schedule(dynamic)
        for (int64_t s = 0; s < nslab; ++s) {
            memset(vr, 0, sizeof(double) * (size_t)nS);
            memset(vi, 0, sizeof(double) * (size_t)nS);
            for (int64_t i0 = 0; i0 < g[0]; ++i0)
                for (int64_t i1 = 0; i1 < g[1]; ++i1)
                    for (int64_t i2 = 0; i2 < g[2]; ++i2)
                        vr[(i0 * S[1] + i1) * S[2] + i2] = v[s * ng + (i0 * g[1] + i1) * g[2] + i2];
            memcpy(kr, Kern + kidx[s] * nS, sizeof(double) * (size_t)nS);
            memset(ki, 0, sizeof(double) * (size_t)nS);
            fref_fft3(S, vr, vi, 0, lr, li);
            fref_fft3(S, kr, ki, 0, lr, li);
            for (int64_t j = 0; j < nS; ++j) {
                const double a = vr[j] * kr[j] - vi[j] * ki[j];
                const double b = vr[j] * ki[j] + vi[j] * kr[j];
                vr[j] = a;
                vi[j] = b;
            }
            fref_fft3(S, vr, vi, 1, lr, li);
            for (int64_t i0 = 0; i0 < g[0]; ++i0)
                for (int64_t i1 = 0; i1 < g[1]; ++i1)
                    for (int64_t i2 = 0; i2 < g[2]; ++i2) {
                        const int64_t o = s * ng + (i0 * g[1] + i1) * g[2] + i2;
                        const double c = vr[(i0 * S[1] + i1) * S[2] + i2] / (double)nS;
                        y[o] = x1 ? x1[o] * c : c;
                    }
        }
        free(vr); free(vi); free(kr); free(ki); free(lr); free(li);
    }
}
