// backward.cu -- element-wise and reduction kernels of the operator's
// backward pass (the FFT convolutions it needs run through the forward
// kernels; see hyena_operator_backward in api.cu).
//
// With z_0 = v, c_k = h_k * z_{k-1} + D_k z_{k-1}, z_k = x_k ⊙ c_k, y = z_K
// ([HN] 아키텍처 상세, step 3) and g_K = dL/dy:
//   dx_k = g_k ⊙ c_k,   e_k = g_k ⊙ x_k,
//   g_{k-1}[s] = Σ_{t>=s} h_k[t-s] e_k[t] + D_k e_k[s],
//   dh_k[τ] = Σ_b Σ_{t>=τ} e_k[t] z_{k-1}[t-τ],   dD_k = Σ_b Σ_t e_k[t] z_{k-1}[t].
// Both sums over t >= s are causal convolutions of the time-reversed e_k:
// these kernels write e_k reversed and read the convolution results back
// reversed.
#include <cuda_bf16.h>

#include "kernels.h"
#include "status.h"

namespace hy {

namespace {

__device__ __forceinline__ float ld_io(const float *p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_io(const __nv_bfloat16 *p, int64_t i) { return __bfloat162float(p[i]); }
__device__ __forceinline__ void st_io(float *p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st_io(__nv_bfloat16 *p, int64_t i, float v) { p[i] = __float2bfloat16_rn(v); }

constexpr int NT = 256;

unsigned grid_for(int64_t n) {
    int64_t b = (n + NT - 1) / NT;
    const int64_t cap = (int64_t)148 * 32;
    return (unsigned)(b < 1 ? 1 : (b > cap ? cap : b));
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_to_f32(const IO *src, float *dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) dst[i] = ld_io(src, i);
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_from_f32(const float *src, IO *dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) st_io(dst, i, src[i]);
}

// z = x ⊙ c
template <typename IO>
__global__ void __launch_bounds__(NT) k_gate(const IO *x, const float *c, float *z, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) z[i] = ld_io(x, i) * c[i];
}

// dx = g ⊙ c; er[row][L-1-t] = g[row][t] x[row][t]
template <typename IO>
__global__ void __launch_bounds__(NT) k_dx_e(const float *g, const float *c, const IO *x, IO *dx, float *er,
                                             int64_t n, int L) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) {
        const float gi = g[i];
        st_io(dx, i, gi * c[i]);
        const int64_t row = i / L, t = i - row * L;
        er[row * L + (L - 1 - t)] = gi * ld_io(x, i);
    }
}

// g[row][t] <- r[row][L-1-t] + D[row % D] g[row][t] x[row][t]  (in place)
template <typename IO>
__global__ void __launch_bounds__(NT) k_next_g(const float *r, float *g, const IO *x, const float *Dk, int64_t n,
                                               int D, int L) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) {
        const int64_t row = i / L, t = i - row * L;
        float v = r[row * L + (L - 1 - t)];
        if (Dk) v = fmaf(__ldg(Dk + row % D), g[i] * ld_io(x, i), v);
        g[i] = v;
    }
}

// dh[d][τ] = Σ_b w[b D + d][L-1-τ]
__global__ void __launch_bounds__(NT) k_dh(const float *w, float *dh, int B, int D, int L) {
    const int64_t n = (int64_t)D * L;
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) {
        const int64_t d = i / L, tau = i - d * L;
        float s = 0.f;
        for (int b = 0; b < B; ++b) s += w[((int64_t)b * D + d) * L + (L - 1 - tau)];
        dh[i] = s;
    }
}

// dD[d] = Σ_b Σ_t g x z over the rows b D + d (one CTA per channel)
template <typename IO>
__global__ void __launch_bounds__(NT) k_dD(const float *g, const IO *x, const float *z, float *dD, int B, int D,
                                           int L) {
    const int d = blockIdx.x;
    float s = 0.f;
    for (int b = 0; b < B; ++b) {
        const int64_t base = ((int64_t)b * D + d) * L;
        for (int t = threadIdx.x; t < L; t += NT) s = fmaf(g[base + t] * ld_io(x, base + t), z[base + t], s);
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __shared__ float part[NT / 32];
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        float tot = 0.f;
        for (int w = 0; w < NT / 32; ++w) tot += part[w];
        dD[d] = tot;
    }
}

}  // namespace

#define HY_IO_DISPATCH(dt, T, ...)                         \
    do {                                                   \
        if ((dt) == HY_BF16) {                             \
            using T = __nv_bfloat16;                       \
            __VA_ARGS__;                                   \
        } else {                                           \
            using T = float;                               \
            __VA_ARGS__;                                   \
        }                                                  \
    } while (0)

hy_status bw_to_f32(const void *src, hy_dtype dt, float *dst, int64_t n, cudaStream_t s) {
    HY_IO_DISPATCH(dt, T, k_to_f32<T><<<grid_for(n), NT, 0, s>>>(reinterpret_cast<const T *>(src), dst, n));
    return check_launch("backward: convert");
}

hy_status bw_from_f32(const float *src, hy_dtype dt, void *dst, int64_t n, cudaStream_t s) {
    HY_IO_DISPATCH(dt, T, k_from_f32<T><<<grid_for(n), NT, 0, s>>>(src, reinterpret_cast<T *>(dst), n));
    return check_launch("backward: convert");
}

hy_status bw_gate(const void *x, hy_dtype dt, const float *c, float *z, int64_t n, cudaStream_t s) {
    HY_IO_DISPATCH(dt, T, k_gate<T><<<grid_for(n), NT, 0, s>>>(reinterpret_cast<const T *>(x), c, z, n));
    return check_launch("backward: gate");
}

hy_status bw_dx_e(const float *g, const float *c, const void *x, hy_dtype dt, void *dx, float *er, int64_t rows, int L,
                  cudaStream_t s) {
    const int64_t n = rows * L;
    HY_IO_DISPATCH(dt, T, k_dx_e<T><<<grid_for(n), NT, 0, s>>>(g, c, reinterpret_cast<const T *>(x),
                                                                reinterpret_cast<T *>(dx), er, n, L));
    return check_launch("backward: dx");
}

hy_status bw_next_g(const float *r, float *g, const void *x, hy_dtype dt, const float *Dk, int64_t rows, int D, int L,
                    cudaStream_t s) {
    const int64_t n = rows * L;
    HY_IO_DISPATCH(dt, T, k_next_g<T><<<grid_for(n), NT, 0, s>>>(r, g, reinterpret_cast<const T *>(x), Dk, n, D, L));
    return check_launch("backward: next gradient");
}

hy_status bw_dh(const float *w, float *dh, int B, int D, int L, cudaStream_t s) {
    k_dh<<<grid_for((int64_t)D * L), NT, 0, s>>>(w, dh, B, D, L);
    return check_launch("backward: dh");
}

hy_status bw_dD(const float *g, const void *x, hy_dtype dt, const float *z, float *dD, int B, int D, int L,
                cudaStream_t s) {
    HY_IO_DISPATCH(dt, T, k_dD<T><<<D, NT, 0, s>>>(g, reinterpret_cast<const T *>(x), z, dD, B, D, L));
    return check_launch("backward: dD");
}

#undef HY_IO_DISPATCH

}  // namespace hy
