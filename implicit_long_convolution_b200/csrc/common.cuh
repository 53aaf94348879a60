// common.cuh -- small shared pieces of the sm_100a library: complex helpers,
// compile-time trigonometry for butterfly constants, status plumbing.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <type_traits>
#include <utility>

#include "../../include/hyena.h"

namespace hy {

// ----------------------------------------------------------------------------
// complex float2 helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
// a * w
__device__ __forceinline__ float2 cmul(float2 a, float2 w) {
    return make_float2(fmaf(a.x, w.x, -a.y * w.y), fmaf(a.x, w.y, a.y * w.x));
}
// a * conj(w)
__device__ __forceinline__ float2 cmulc(float2 a, float2 w) {
    return make_float2(fmaf(a.x, w.x, a.y * w.y), fmaf(a.y, w.x, -a.x * w.y));
}
// a * w for DIR = -1, a * conj(w) for DIR = +1 (w holds the forward twiddle)
template <int DIR>
__device__ __forceinline__ float2 cmul_dir(float2 a, float2 w) {
    if constexpr (DIR < 0) return cmul(a, w);
    else return cmulc(a, w);
}

// f(integral_constant<int, I>) for I in the sequence, in order
template <typename F, int... I>
__device__ __forceinline__ void fold_seq(F &&f, std::integer_sequence<int, I...>) {
    (f(std::integral_constant<int, I>{}), ...);
}

// ----------------------------------------------------------------------------
// compile-time trig (Taylor series on |x| <= pi, evaluated in double)
// ----------------------------------------------------------------------------
__host__ __device__ constexpr double ct_pi() { return 3.14159265358979323846264338327950288; }

__host__ __device__ constexpr double ct_cos(double x) {
    double term = 1.0, sum = 1.0;
    for (int n = 1; n < 32; ++n) {
        term *= -x * x / ((2.0 * n - 1.0) * (2.0 * n));
        sum += term;
    }
    return sum;
}
__host__ __device__ constexpr double ct_sin(double x) {
    double term = x, sum = x;
    for (int n = 1; n < 32; ++n) {
        term *= -x * x / ((2.0 * n) * (2.0 * n + 1.0));
        sum += term;
    }
    return sum;
}
// angle 2*pi*e/N reduced to [-pi, pi]
__host__ __device__ constexpr double ct_angle(int e, int N) {
    int r = ((e % N) + N) % N;
    if (2 * r > N) r -= N;
    return 2.0 * ct_pi() * (double)r / (double)N;
}

// v * W_N^E with W_N = exp(DIR * 2*pi*i / N)  (DIR = -1 forward, +1 inverse)
template <int DIR, int N, int E>
__device__ __forceinline__ float2 rot(float2 v) {
    constexpr int e = ((E % N) + N) % N;
    if constexpr (e == 0) {
        return v;
    } else if constexpr (2 * e == N) {
        return make_float2(-v.x, -v.y);
    } else if constexpr (4 * e == N) {          // W = DIR * i
        if constexpr (DIR < 0) return make_float2(v.y, -v.x);
        else return make_float2(-v.y, v.x);
    } else if constexpr (4 * e == 3 * N) {      // W = -DIR * i
        if constexpr (DIR < 0) return make_float2(-v.y, v.x);
        else return make_float2(v.y, -v.x);
    } else if constexpr (8 * e == N || 8 * e == 3 * N || 8 * e == 5 * N || 8 * e == 7 * N) {
        // W = (c + i s) with |c| = |s| = 1/sqrt(2)
        constexpr float h = 0.70710678118654752440f;
        constexpr double ang = ct_angle(e, N);
        constexpr float c = ct_cos(ang) > 0 ? h : -h;
        constexpr float s = (DIR * ct_sin(ang)) > 0 ? h : -h;
        if constexpr (c == s) {
            return make_float2((v.x - v.y) * c, (v.x + v.y) * c);
        } else {
            // c = -s
            return make_float2((v.x + v.y) * c, (v.y - v.x) * c);
        }
    } else {
        constexpr double ang = ct_angle(e, N);
        constexpr float c = (float)ct_cos(ang);
        constexpr float s = (float)(DIR * ct_sin(ang));
        return make_float2(fmaf(v.x, c, -v.y * s), fmaf(v.x, s, v.y * c));
    }
}

// ----------------------------------------------------------------------------
// Ordered read-only global loads.  Volatile asm keeps each load where it is
// written: the compiler neither hoists it above the barriers of an FFT (which
// would hold a register per in-flight value through the transform) nor
// speculates it out of the branch that guards it.
// ----------------------------------------------------------------------------
// Streaming data (signals, spectra) is read once per SM: L1::no_allocate keeps
// it from evicting the twiddle tables, which every row re-reads.
__device__ __forceinline__ float ldv(const float *p) {
    float v;
    asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ float2 ldv(const float2 *p) {
    float2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldv_u16(const void *p) {
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ uint32_t ldv_u32(const void *p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
__device__ __forceinline__ float4 ldv4(const float *p) {
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ uint2 ldv_u64(const void *p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}
// L1-cached ordered load (small tables shared by all rows)
__device__ __forceinline__ float2 ldc(const float2 *p) {
    float2 v;
    asm volatile("ld.global.nc.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "l"(p));
    return v;
}

// ----------------------------------------------------------------------------
// IO element types (fp32 or bfloat16 in memory, fp32 in registers)
// ----------------------------------------------------------------------------
template <typename IO> struct IOTraits;
template <> struct IOTraits<float> {
    static __device__ __forceinline__ float load(const float *p) { return ldv(p); }
    static __device__ __forceinline__ float2 load2(const float *p) {
        return ldv(reinterpret_cast<const float2 *>(p));
    }
    // 4 consecutive elements; p 16-byte aligned
    static __device__ __forceinline__ float4 load4(const float *p) { return ldv4(p); }
    static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
    static __device__ __forceinline__ void store2(float *p, float2 v) {
        *reinterpret_cast<float2 *>(p) = v;
    }
    static __device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
};
// bf16 -> fp32 is the exact widening of the top 16 bits.
template <> struct IOTraits<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
        return __uint_as_float(ldv_u16(p) << 16);
    }
    static __device__ __forceinline__ float2 load2(const __nv_bfloat16 *p) {
        const uint32_t v = ldv_u32(p);
        return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
    }
    // 4 consecutive elements; p 8-byte aligned
    static __device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
        const uint2 v = ldv_u64(p);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }
    static __device__ __forceinline__ void store2(__nv_bfloat16 *p, float2 v) {
        *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(v.x, v.y);
    }
    static __device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
        uint2 u;
        u.x = *reinterpret_cast<const uint32_t *>(&a);
        u.y = *reinterpret_cast<const uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = u;
    }
};

}  // namespace hy
