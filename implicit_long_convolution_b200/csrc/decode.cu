// decode.cu -- streaming decode step of the spectral gate with a prefix-FFT
// cache ([SP] 토큰 믹서 구성과 생성 지원: the cache plays the role of a
// KV-cache, so autoregressive generation does not redo the FFT each step).
//
// The cache holds, for every row, the spectrum of the prefix seen so far on
// the n/2 + 1 bins of the length-n transform (later positions zero):
//   X_k <- X_k + x[pos] e^{-2πi k pos / n}            (the new token)
//   y[pos] = x2[pos] · (1/n) Σ_k c_k Re(G_k X_k e^{+2πi k pos / n}),
// c_0 = c_{n/2} = 1, c_k = 2 otherwise -- the inverse real transform of the
// gated prefix spectrum at the one new position (only the real part of the
// product counts at DC and Nyquist, as in the spectral gate).  One CTA per
// row; each step reads and writes the row's cache once: O(n) per token
// instead of the O(n log n) of a full transform.  A thread's bins are NT
// apart, so its twiddles advance by the fixed rotation e^{2πi NT pos/n},
// recomputed exactly every 8th bin.
#include <cuda_bf16.h>

#include "kernels.h"
#include "status.h"

namespace hy {

namespace {

constexpr int NT = 256;

__device__ __forceinline__ float ld1(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld1(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st1(float *p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st1(__nv_bfloat16 *p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

template <typename IO>
__global__ void __launch_bounds__(NT) gate_decode_kernel(const GateDecodeArgs a, const IO *x, const IO *x2, IO *y) {
    const int nb = a.n / 2 + 1;
    const uint64_t mask = (uint64_t)a.n - 1;
    for (int64_t row = blockIdx.x; row < a.rows; row += gridDim.x) {
        const float xv = ld1(x, row);
        const float2 *G = a.g + (row / (a.dh * a.heads)) * a.g_batch_stride + ((row / a.dh) % a.heads) * (int64_t)nb;
        float2 *X = a.cache + row * (int64_t)nb;
        float acc = 0.f;
        // this thread's bins k, k + NT, ...: W^{(k + NT) pos} = W^{k pos} W^{NT pos};
        // exact every 8th bin, the step rotation in between (a few ulp).
        // Bins go in groups of U whose cache and gate loads are all issued
        // before any of them is used.
        constexpr int U = 8;
        float s1, c1;
        sincospif((float)(2 * (((uint64_t)NT * (uint64_t)a.pos) & mask)) / (float)a.n, &s1, &c1);
        float s = 0.f, c = 1.f;
        int j = 0;
        for (int k0 = threadIdx.x; k0 < nb; k0 += U * NT) {
            float2 Xk[U], gk[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int k = k0 + u * NT;
                if (k < nb) {
                    Xk[u] = X[k];
                    gk[u] = __ldg(G + k);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u, ++j) {
                const int k = k0 + u * NT;
                if (k >= nb) break;
                if ((j & 7) == 0) {
                    const uint64_t m = ((uint64_t)k * (uint64_t)a.pos) & mask;   // k pos mod n, exact
                    sincospif((float)(2 * m) / (float)a.n, &s, &c);             // W = e^{+2πi m/n} = (c, s)
                } else {
                    const float cn = c * c1 - s * s1;
                    s = fmaf(s, c1, c * s1);
                    c = cn;
                }
                float2 v = Xk[u];
                v.x = fmaf(xv, c, v.x);                                          // + x conj(W)
                v.y = fmaf(-xv, s, v.y);
                X[k] = v;
                const float pr = gk[u].x * v.x - gk[u].y * v.y;                  // P = G X
                const float pi = gk[u].x * v.y + gk[u].y * v.x;
                const float w = (k == 0 || k == nb - 1) ? 1.f : 2.f;
                acc = fmaf(w, pr * c - pi * s, acc);                             // c_k Re(P W)
            }
        }
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        __shared__ float part[NT / 32];
        if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float tot = 0.f;
            for (int i = 0; i < NT / 32; ++i) tot += part[i];
            float v = tot / (float)a.n;
            if (x2) v *= ld1(x2, row);
            st1(y, row, v);
        }
        __syncthreads();   // part[] is reused by the next row
    }
}

}  // namespace

hy_status launch_gate_decode(const GateDecodeArgs &a, hy_dtype dt, const void *x, const void *x2, void *y,
                             cudaStream_t s) {
    int sms = 148, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = a.rows < (int64_t)sms * 8 ? a.rows : (int64_t)sms * 8;
    if (dt == HY_BF16)
        gate_decode_kernel<__nv_bfloat16><<<(unsigned)blocks, NT, 0, s>>>(
            a, reinterpret_cast<const __nv_bfloat16 *>(x), reinterpret_cast<const __nv_bfloat16 *>(x2),
            reinterpret_cast<__nv_bfloat16 *>(y));
    else
        gate_decode_kernel<float><<<(unsigned)blocks, NT, 0, s>>>(a, reinterpret_cast<const float *>(x),
                                                                   reinterpret_cast<const float *>(x2),
                                                                   reinterpret_cast<float *>(y));
    return check_launch("spectral_gate_decode launch");
}

}  // namespace hy
