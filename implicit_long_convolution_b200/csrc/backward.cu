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

// 4 consecutive elements (16 bytes of fp32, 8 of bf16)
__device__ __forceinline__ float4 ld4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}
__device__ __forceinline__ void st4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<const uint32_t *>(&a);
    u.y = *reinterpret_cast<const uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
}
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 rev4(float4 a) { return make_float4(a.w, a.z, a.y, a.x); }

constexpr int NT = 256;

unsigned grid_for(int64_t n) {
    int64_t b = (n + NT - 1) / NT;
    const int64_t cap = (int64_t)148 * 32;
    return (unsigned)(b < 1 ? 1 : (b > cap ? cap : b));
}

// Element-wise passes walk rows: block y strides over rows, threads over
// the row in groups of 4 (L a multiple of 4) or singly.
#define HY_ROWS_LOOP(rows)                                                        \
    for (int64_t row = blockIdx.y; row < (rows); row += gridDim.y)

dim3 rows_grid(int64_t rows, int L, bool vec) {
    const int per_row = (vec ? L / 4 : L);
    unsigned x = (unsigned)((per_row + NT - 1) / NT);
    if (x < 1) x = 1;
    int64_t y = (int64_t)148 * 64 / x;
    if (y < 1) y = 1;
    if (y > rows) y = rows;
    if (y > 65535) y = 65535;
    return dim3(x, (unsigned)y);
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_to_f32(const IO *src, float *dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) dst[i] = ld_io(src, i);
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_to_f32_v(const IO *src, float *dst, int64_t n4) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n4; i += (int64_t)gridDim.x * NT)
        st4(dst + 4 * i, ld4(src + 4 * i));
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_from_f32(const float *src, IO *dst, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) st_io(dst, i, src[i]);
}

template <typename IO>
__global__ void __launch_bounds__(NT) k_from_f32_v(const float *src, IO *dst, int64_t n4) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n4; i += (int64_t)gridDim.x * NT)
        st4(dst + 4 * i, ld4(src + 4 * i));
}

// z = x ⊙ c
template <typename IO>
__global__ void __launch_bounds__(NT) k_gate(const IO *x, const float *c, float *z, int64_t n) {
    for (int64_t i = blockIdx.x * (int64_t)NT + threadIdx.x; i < n; i += (int64_t)gridDim.x * NT) z[i] = ld_io(x, i) * c[i];
}

// dx = g ⊙ c; er[row][L-1-t] = g[row][t] x[row][t]
template <typename IO, bool VEC>
__global__ void __launch_bounds__(NT) k_dx_e(const float *g, const float *c, const IO *x, IO *dx, float *er,
                                             int64_t rows, int L) {
    HY_ROWS_LOOP(rows) {
        const int64_t o = row * L;
        if constexpr (VEC) {
            for (int q = blockIdx.x * NT + threadIdx.x; q < L / 4; q += gridDim.x * NT) {
                const int t = 4 * q;
                const float4 gv = ld4(g + o + t);
                st4(dx + o + t, mul4(gv, ld4(c + o + t)));
                st4(er + o + (L - 4 - t), rev4(mul4(gv, ld4(x + o + t))));
            }
        } else {
            for (int t = blockIdx.x * NT + threadIdx.x; t < L; t += gridDim.x * NT) {
                const float gi = g[o + t];
                st_io(dx, o + t, gi * c[o + t]);
                er[o + (L - 1 - t)] = gi * ld_io(x, o + t);
            }
        }
    }
}

// g[row][t] <- r[row][L-1-t] + D[row % D] g[row][t] x[row][t]  (in place)
template <typename IO, bool VEC>
__global__ void __launch_bounds__(NT) k_next_g(const float *r, float *g, const IO *x, const float *Dk, int64_t rows,
                                               int D, int L) {
    HY_ROWS_LOOP(rows) {
        const int64_t o = row * L;
        const float dk = Dk ? __ldg(Dk + row % D) : 0.f;
        if constexpr (VEC) {
            for (int q = blockIdx.x * NT + threadIdx.x; q < L / 4; q += gridDim.x * NT) {
                const int t = 4 * q;
                const float4 rv = rev4(ld4(r + o + (L - 4 - t)));
                const float4 e = mul4(ld4(g + o + t), ld4(x + o + t));
                st4(g + o + t, make_float4(fmaf(dk, e.x, rv.x), fmaf(dk, e.y, rv.y), fmaf(dk, e.z, rv.z),
                                           fmaf(dk, e.w, rv.w)));
            }
        } else {
            for (int t = blockIdx.x * NT + threadIdx.x; t < L; t += gridDim.x * NT)
                g[o + t] = fmaf(dk, g[o + t] * ld_io(x, o + t), r[o + (L - 1 - t)]);
        }
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

// Vector paths need 4 | n and row starts at a multiple of 4 elements; the
// pointers are the library's own workspace or the caller's signals, whose
// alignment the entry point checks (16-byte fp32 / 8-byte bf16 when 4 | L).
hy_status bw_to_f32(const void *src, hy_dtype dt, float *dst, int64_t n, cudaStream_t s) {
    const bool vec = n % 4 == 0 && (uintptr_t)src % (4 * (dt == HY_BF16 ? 2 : 4)) == 0;
    if (vec)
        HY_IO_DISPATCH(dt, T, k_to_f32_v<T><<<grid_for(n / 4), NT, 0, s>>>(reinterpret_cast<const T *>(src), dst, n / 4));
    else
        HY_IO_DISPATCH(dt, T, k_to_f32<T><<<grid_for(n), NT, 0, s>>>(reinterpret_cast<const T *>(src), dst, n));
    return check_launch("backward: convert");
}

hy_status bw_from_f32(const float *src, hy_dtype dt, void *dst, int64_t n, cudaStream_t s) {
    const bool vec = n % 4 == 0 && (uintptr_t)dst % (4 * (dt == HY_BF16 ? 2 : 4)) == 0;
    if (vec)
        HY_IO_DISPATCH(dt, T, k_from_f32_v<T><<<grid_for(n / 4), NT, 0, s>>>(src, reinterpret_cast<T *>(dst), n / 4));
    else
        HY_IO_DISPATCH(dt, T, k_from_f32<T><<<grid_for(n), NT, 0, s>>>(src, reinterpret_cast<T *>(dst), n));
    return check_launch("backward: convert");
}

hy_status bw_gate(const void *x, hy_dtype dt, const float *c, float *z, int64_t n, cudaStream_t s) {
    HY_IO_DISPATCH(dt, T, k_gate<T><<<grid_for(n), NT, 0, s>>>(reinterpret_cast<const T *>(x), c, z, n));
    return check_launch("backward: gate");
}

hy_status bw_dx_e(const float *g, const float *c, const void *x, hy_dtype dt, void *dx, float *er, int64_t rows, int L,
                  cudaStream_t s) {
    const size_t al = 4 * (dt == HY_BF16 ? 2 : 4);
    const bool vec = L % 4 == 0 && (uintptr_t)x % al == 0 && (uintptr_t)dx % al == 0;
    const dim3 grid = rows_grid(rows, L, vec);
    if (vec)
        HY_IO_DISPATCH(dt, T, k_dx_e<T, true><<<grid, NT, 0, s>>>(g, c, reinterpret_cast<const T *>(x),
                                                                   reinterpret_cast<T *>(dx), er, rows, L));
    else
        HY_IO_DISPATCH(dt, T, k_dx_e<T, false><<<grid, NT, 0, s>>>(g, c, reinterpret_cast<const T *>(x),
                                                                    reinterpret_cast<T *>(dx), er, rows, L));
    return check_launch("backward: dx");
}

hy_status bw_next_g(const float *r, float *g, const void *x, hy_dtype dt, const float *Dk, int64_t rows, int D, int L,
                    cudaStream_t s) {
    const size_t al = 4 * (dt == HY_BF16 ? 2 : 4);
    const bool vec = L % 4 == 0 && (uintptr_t)x % al == 0;
    const dim3 grid = rows_grid(rows, L, vec);
    if (vec)
        HY_IO_DISPATCH(dt, T, k_next_g<T, true><<<grid, NT, 0, s>>>(r, g, reinterpret_cast<const T *>(x), Dk, rows, D, L));
    else
        HY_IO_DISPATCH(dt, T, k_next_g<T, false><<<grid, NT, 0, s>>>(r, g, reinterpret_cast<const T *>(x), Dk, rows, D, L));
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
