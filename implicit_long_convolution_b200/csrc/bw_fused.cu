// bw_fused.cu -- backward pass of the order-2 operator, fused per channel on
// chip ([HN] 아키텍처 상세, step 3, differentiated).
//
// For channel d and its B rows (b, d), with y = x_1 ⊙ (h * v + D v):
//   c   = h * v + D v                   C  = X(v) (H + D)
//   dx1 = dy ⊙ c
//   e   = dy ⊙ x1
//   dv[s] = Σ_{t>=s} h[t-s] e[t] + D e[s]      DV = X(e) conj(H + D)
//   dh[τ] = Σ_b Σ_{t>=τ} e_b[t] v_b[t-τ]        DH = Σ_b X(e_b) conj(X(v_b))
//   dD    = Σ_b Σ_t e_b[t] v_b[t]
// where X() is the real DFT of a row zero-padded to n = 2L.  The two sums
// over t >= s are correlations: conj() of a real row's spectrum is the
// spectrum of the row reversed modulo n, and with the padding to 2L the
// wrapped-around part multiplies zeros, so no row is reversed in memory.
//
// One persistent CTA takes a channel at a time and walks its B rows: per row
// the forward transforms of e and v (packed complex FFT of M = n/2 points and
// the real-FFT split, as in the forward kernels), the two products, their
// merges and inverse transforms (dx1 and dv written out), and the running
// batch sum X(e) conj(X(v)) kept in shared memory; after the channel's last
// row one more merge and inverse transform give dh, and a block reduction
// gives dD.  The B D rows are dealt out in channel-major order as equal
// contiguous ranges (at least B rows each), so a channel is shared by at most
// two CTAs; each adds its share of dh and dD onto the zeroed outputs with
// atomicAdd, and as fp32 addition of two terms onto zero commutes, the result
// does not depend on which CTA comes first.  X(e) waits in shared memory
// while X(v) is formed, so a thread holds one packed row at a time; the next
// row's v, x1 and dy are asked into L2 (bulk prefetch) while the current row
// is transformed, and read with plain coalesced loads.
#include <cuda_bf16.h>

#include "../../include/hyena.h"
#include "common.cuh"
#include "fft_core.cuh"
#include "kernels.h"
#include "resident.cuh"
#include "status.h"
#include "twiddle.h"

namespace hy {

namespace {

struct BwParams {
    int B, D;
    const void *v, *x1, *dy;   // (B, D, L), L = M samples per row
    const float2 *H;           // (D, M + 1) spectrum of h
    const float *Dsk;          // (D) or NULL
    void *dv, *dx1;            // (B, D, L)
    float *dh;                 // (D, L) or NULL
    float *dD;                 // (D) or NULL
    float scale;               // 1 / (2n)
    const float2 *tw_fft;
    const float2 *tw_split;
};

// 16 points per thread (512 threads at M = 8192, 16 warps on an SM, 128
// registers per thread).
__host__ __device__ constexpr int bw_log_p(int log_m) { return log_m - 5 < 2 ? 2 : (log_m - 5 > 4 ? 4 : log_m - 5); }
__host__ __device__ constexpr int bw_threads(int log_m) { return (1 << log_m) >> bw_log_p(log_m); }
// shared memory: FFT exchange buffer, the batch sum and the stash of X(e)
// (M + 1 bins each)
__host__ __device__ constexpr size_t bw_acc_offset(int log_m) { return (size_t)stream_stage_offset(1 << log_m); }
__host__ __device__ constexpr size_t bw_bins_slots(int log_m) { return (size_t)(((1 << log_m) + 2) / 2) * 2; }
__host__ __device__ constexpr size_t bw_stash_offset(int log_m) { return bw_acc_offset(log_m) + bw_bins_slots(log_m); }
__host__ __device__ constexpr size_t bw_smem_bytes(int log_m) {
    return (bw_stash_offset(log_m) + bw_bins_slots(log_m)) * 8;
}

// Real-FFT split of a packed spectrum held in the own layout (x[m] = Z[t + m T]):
// afterwards x[m] = 2 X[k] and x[P/2 + m] = 2 X[M - k] for k = t + m T, m < P/2,
// and (thread 0) mid = 2 X[M/2].  X[0] and X[M] are real.
template <int LOG_M, int LOG_P>
__device__ __forceinline__ void split_pairs(float2 (&x)[1 << LOG_P], float2 &mid, float2 *sbuf, int t,
                                            const float2 *__restrict__ tws) {
    constexpr int P = 1 << LOG_P;
    store_own<LOG_M, LOG_P>(x, sbuf, t);
    const float2 wt0 = ldc(tws + t);
    mid = make_float2(2.f * x[P / 2].x, -2.f * x[P / 2].y);   // X[M/2] = conj Z[M/2]
    __syncthreads();
    float2 xn[P / 2];
    auto pair = [&](auto mc) {
        constexpr int m = decltype(mc)::value;
        if (m == 0 && t == 0) {
            const float2 z0 = x[0];
            x[0] = make_float2(2.f * (z0.x + z0.y), 0.f);
            xn[0] = make_float2(2.f * (z0.x - z0.y), 0.f);
        } else {
            const float2 zk = x[m];
            const float2 zn = sbuf[partner_slot<LOG_M, LOG_P>(t, m)];
            const float2 A = make_float2(zk.x + zn.x, zk.y - zn.y);   // Z[k] + Z*[M-k]
            const float2 Bv = make_float2(zk.x - zn.x, zk.y + zn.y);  // Z[k] - Z*[M-k]
            const float2 wB = cmul(Bv, rot<-1, 2 * P, m>(wt0));       // W_n^k B
            const float2 C = make_float2(wB.y, -wB.x);                // -i W B
            x[m] = cadd(A, C);
            xn[m] = cconj(csub(A, C));
        }
    };
    fold_seq(pair, std::make_integer_sequence<int, P / 2>{});
#pragma unroll
    for (int m = 0; m < P / 2; ++m) x[P / 2 + m] = xn[m];
    __syncthreads();
}

// Inverse of split_pairs for a product spectrum Y in the same pair layout
// (x[m] = Y[k], x[P/2 + m] = Y[M - k], mid = Y[M/2] in thread 0, Y[0] and
// Y[M] real): afterwards x holds the packed spectrum (own layout) whose
// inverse FFT times the usual 1/(2n) is the real row.
template <int LOG_M, int LOG_P>
__device__ __forceinline__ void merge_pairs(float2 (&x)[1 << LOG_P], float2 mid, float2 *sbuf, int t,
                                            const float2 *__restrict__ tws) {
    constexpr int P = 1 << LOG_P;
    const float2 wt0 = ldc(tws + t);
    auto pair = [&](auto mc) {
        constexpr int m = decltype(mc)::value;
        const float2 yk = x[m], yn = x[P / 2 + m];
        if (m == 0 && t == 0) {
            x[0] = make_float2(yk.x + yn.x, yk.x - yn.x);           // DC and Nyquist, real
        } else {
            const float2 A2 = make_float2(yk.x + yn.x, yk.y - yn.y);
            const float2 B2 = make_float2(yk.x - yn.x, yk.y + yn.y);
            const float2 cB = cmulc(B2, rot<-1, 2 * P, m>(wt0));    // W_n^{-k} B
            const float2 C2 = make_float2(-cB.y, cB.x);
            x[m] = cadd(A2, C2);
            sbuf[partner_slot<LOG_M, LOG_P>(t, m)] = cconj(csub(A2, C2));
        }
    };
    fold_seq(pair, std::make_integer_sequence<int, P / 2>{});
    if (t == 0) x[P / 2] = make_float2(2.f * mid.x, -2.f * mid.y);   // Z'[M/2] = 2 conj Y[M/2]
    __syncthreads();
#pragma unroll
    for (int m = P / 2; m < P; ++m)
        if (!(t == 0 && m == P / 2)) x[m] = sbuf[own_slot<LOG_M, LOG_P>(t, m)];
    __syncthreads();
}

template <int LOG_M, typename IO>
__global__ void __launch_bounds__(bw_threads(LOG_M), bw_threads(LOG_M) >= 512 ? 1 : 512 / bw_threads(LOG_M)) bw_fused_kernel(const BwParams p) {
    constexpr int LOG_P = bw_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int PIN = P / 2;                               // packed points carrying samples
    constexpr uint32_t ROW_BYTES = (uint32_t)(M * sizeof(IO));
    static_assert(ROW_BYTES % 16 == 0, "bulk prefetch size");
    using IOT = IOTraits<IO>;

    extern __shared__ __align__(128) float2 smem[];
    float2 *sbuf = smem;
    float2 *acc = smem + bw_acc_offset(LOG_M);               // [P][T] pair layout, then bin M/2
    float2 *es = smem + bw_stash_offset(LOG_M);              // X(e) of the row, same layout
    __shared__ float red[32];

    const int t = threadIdx.x;
    const int B = p.B, D = p.D;
    const IO *vb = reinterpret_cast<const IO *>(p.v);
    const IO *xb = reinterpret_cast<const IO *>(p.x1);
    const IO *gb = reinterpret_cast<const IO *>(p.dy);
    IO *dvb = reinterpret_cast<IO *>(p.dv);
    IO *dxb = reinterpret_cast<IO *>(p.dx1);
    // rows in channel-major order q = d B + b; this CTA takes [q0, q1), at
    // least B rows, so a channel is split between at most two CTAs
    const int64_t R = (int64_t)B * D;
    const int64_t q0 = (int64_t)blockIdx.x * R / gridDim.x, q1 = (int64_t)(blockIdx.x + 1) * R / gridDim.x;
    auto row_of = [&](int64_t q) { return (q % B) * (int64_t)D + q / B; };
    float dpart = 0.f;
    for (int64_t q = q0; q < q1; ++q) {
        const int b = (int)(q % B);
        const int64_t d = q / B;
        const int64_t row = (int64_t)b * D + d;
        const bool seg_start = b == 0 || q == q0, seg_end = b == B - 1 || q == q1 - 1;
        // the next row's inputs are asked into L2 while this one is transformed
        if (t == 0) {
            const int64_t nrow = q + 1 < q1 ? row_of(q + 1) : -1;
            if (nrow >= 0) {
                bulk_prefetch_l2(vb + nrow * M, ROW_BYTES);
                bulk_prefetch_l2(xb + nrow * M, ROW_BYTES);
                bulk_prefetch_l2(gb + nrow * M, ROW_BYTES);
            }
        }
        // e = dy ⊙ x1 and the dD sum; v is read again for its own transform
        // (an L2 hit), so only one packed row is live during each transform
        float2 xe[P];
#pragma unroll
        for (int m = 0; m < P; ++m) xe[m] = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < PIN; ++m) {
            const int64_t i0 = row * M + 2 * (t + m * T);
            const float2 a = IOT::load2(vb + i0), x1 = IOT::load2(xb + i0), g = IOT::load2(gb + i0);
            const float2 e = make_float2(g.x * x1.x, g.y * x1.y);
            xe[m] = e;
            dpart = fmaf(e.x, a.x, fmaf(e.y, a.y, dpart));
        }
        if (seg_start && p.dh) {
#pragma unroll
            for (int j = 0; j < P; ++j) acc[j * T + t] = make_float2(0.f, 0.f);
            if (t == 0) acc[M] = make_float2(0.f, 0.f);
        }
        // ---- X(e) to the stash, then X(v) in registers (pair layout)
        float2 emid, vmid;
        block_fft<LOG_M, LOG_P, -1, true>(xe, sbuf, t, p.tw_fft);
        split_pairs<LOG_M, LOG_P>(xe, emid, sbuf, t, p.tw_split);
#pragma unroll
        for (int j = 0; j < P; ++j) es[j * T + t] = xe[j];
        float2 xv[P];
#pragma unroll
        for (int m = 0; m < P; ++m) xv[m] = m < PIN ? IOT::load2(vb + row * M + 2 * (t + m * T)) : make_float2(0.f, 0.f);
        block_fft<LOG_M, LOG_P, -1, true>(xv, sbuf, t, p.tw_fft);
        split_pairs<LOG_M, LOG_P>(xv, vmid, sbuf, t, p.tw_split);
        // ---- batch sum of X(e) conj X(v) (own slots only)
        if (p.dh) {
#pragma unroll
            for (int j = 0; j < P; ++j) acc[j * T + t] = cadd(acc[j * T + t], cmulc(es[j * T + t], xv[j]));
            if (t == 0) acc[M] = cadd(acc[M], cmulc(emid, vmid));
        }
        // ---- c = IFFT(X(v) (H + D)), dx1 = dy ⊙ c
        const float dk = p.Dsk ? __ldg(p.Dsk + d) : 0.f;
        const float2 *Hd = p.H + d * (int64_t)(M + 1);
        float2 hmid = ldv(Hd + M / 2);
        hmid.x += dk;
#pragma unroll
        for (int m = 0; m < P / 2; ++m) {
            const int k = t + m * T;
            float2 hk = ldv(Hd + k), hn = ldv(Hd + (M - k));
            hk.x += dk;
            hn.x += dk;
            if (m == 0 && t == 0) {                          // DC and Nyquist: real parts
                xv[0] = make_float2(xv[0].x * hk.x, 0.f);
                xv[P / 2] = make_float2(xv[P / 2].x * hn.x, 0.f);
            } else {
                xv[m] = cmul(xv[m], hk);
                xv[P / 2 + m] = cmul(xv[P / 2 + m], hn);
            }
        }
        merge_pairs<LOG_M, LOG_P>(xv, cmul(vmid, hmid), sbuf, t, p.tw_split);
        block_fft<LOG_M, LOG_P, +1, false>(xv, sbuf, t, p.tw_fft);
#pragma unroll
        for (int m = 0; m < PIN; ++m) {
            const int64_t i0 = row * M + 2 * (t + m * T);
            const float2 g = IOT::load2(gb + i0);            // dy again (an L2 hit)
            IOT::store2(dxb + i0, make_float2(g.x * (xv[m].x * p.scale), g.y * (xv[m].y * p.scale)));
        }
        // ---- dv = IFFT(X(e) conj(H + D))
#pragma unroll
        for (int m = 0; m < P / 2; ++m) {
            const int k = t + m * T;
            float2 hk = ldv(Hd + k), hn = ldv(Hd + (M - k));
            hk.x += dk;
            hn.x += dk;
            const float2 ek = es[m * T + t], en = es[(P / 2 + m) * T + t];
            if (m == 0 && t == 0) {
                xe[0] = make_float2(ek.x * hk.x, 0.f);
                xe[P / 2] = make_float2(en.x * hn.x, 0.f);
            } else {
                xe[m] = cmulc(ek, hk);                       // X(e) conj(H + D)
                xe[P / 2 + m] = cmulc(en, hn);
            }
        }
        merge_pairs<LOG_M, LOG_P>(xe, cmulc(emid, hmid), sbuf, t, p.tw_split);
        block_fft<LOG_M, LOG_P, +1, false>(xe, sbuf, t, p.tw_fft);
#pragma unroll
        for (int m = 0; m < PIN; ++m) {
            const int64_t i0 = row * M + 2 * (t + m * T);
            IOT::store2(dvb + i0, make_float2(xe[m].x * p.scale, xe[m].y * p.scale));
        }
        if (!seg_end) continue;
        // ---- end of this CTA's part of the channel: its share of dD and dh
        //      added onto the zeroed outputs (at most two shares per element)
        if (p.dD) {
            float sum = dpart;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if ((t & 31) == 0) red[t >> 5] = sum;
            __syncthreads();
            if (t == 0) {
                float tot = 0.f;
                for (int w = 0; w < T / 32; ++w) tot += red[w];
                atomicAdd(p.dD + d, tot);
            }
        }
        dpart = 0.f;
        if (p.dh) {
#pragma unroll
            for (int j = 0; j < P; ++j) xe[j] = acc[j * T + t];
            merge_pairs<LOG_M, LOG_P>(xe, t == 0 ? acc[M] : make_float2(0.f, 0.f), sbuf, t, p.tw_split);
            block_fft<LOG_M, LOG_P, +1, false>(xe, sbuf, t, p.tw_fft);
            float *out = p.dh + d * (int64_t)M;
            const float sc = 0.5f * p.scale;                 // both spectra carry the split's factor 2
#pragma unroll
            for (int m = 0; m < PIN; ++m) {
                const int i0 = 2 * (t + m * T);
                atomicAdd(reinterpret_cast<float2 *>(out + i0), make_float2(xe[m].x * sc, xe[m].y * sc));
            }
        }
        __syncthreads();                                     // red[] is reused by the next channel
    }
}

template <int LOG_M, typename IO>
hy_status launch_bw_t(BwParams p, cudaStream_t s) {
    constexpr int T = bw_threads(LOG_M);
    p.tw_fft = tw_stages(LOG_M, bw_log_p(LOG_M));
    p.tw_split = tw_split(LOG_M);
    if (!p.tw_fft || !p.tw_split) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^%d", LOG_M);
    p.scale = (float)(1.0 / (4.0 * (double)(1 << LOG_M)));
    const size_t smem = bw_smem_bytes(LOG_M);
    auto kernel = bw_fused_kernel<LOG_M, IO>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return set_cuda_error("fused backward smem attribute", e);
    }
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, T, smem);
    if (e != cudaSuccess) return set_cuda_error("occupancy query", e);
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)per_sm * device_sm_count();
    if (grid > p.D) grid = p.D;   // at least B rows per CTA
    if (p.dh) {
        cudaError_t e2 = cudaMemsetAsync(p.dh, 0, sizeof(float) * (size_t)p.D * (1 << LOG_M), s);
        if (e2 != cudaSuccess) return set_cuda_error("fused backward dh clear", e2);
    }
    if (p.dD) {
        cudaError_t e2 = cudaMemsetAsync(p.dD, 0, sizeof(float) * (size_t)p.D, s);
        if (e2 != cudaSuccess) return set_cuda_error("fused backward dD clear", e2);
    }
    kernel<<<(unsigned)grid, T, smem, s>>>(p);
    return check_launch("fused backward launch");
}

}  // namespace

bool bw_fused_eligible(int order, int L, hy_dtype dt, const void *const *ptrs16, int nptrs) {
    if (order != 2 || L < 512 || L > 8192 || (L & (L - 1))) return false;
    const int log_m = 31 - __builtin_clz((unsigned)L);
    (void)dt;
    if (bw_smem_bytes(log_m) > (size_t)227 * 1024) return false;
    for (int i = 0; i < nptrs; ++i)
        if (((uintptr_t)ptrs16[i] & 15u) != 0) return false;
    return true;
}

hy_status launch_bw_fused(int B, int D, int L, hy_dtype dt, const void *v, const void *x1, const void *dy,
                          const void *H, const float *Dsk, void *dv, void *dx1, float *dh, float *dD,
                          cudaStream_t s) {
    BwParams p{};
    p.B = B;
    p.D = D;
    p.v = v;
    p.x1 = x1;
    p.dy = dy;
    p.H = reinterpret_cast<const float2 *>(H);
    p.Dsk = Dsk;
    p.dv = dv;
    p.dx1 = dx1;
    p.dh = dh;
    p.dD = dD;
    const bool bf = dt == HY_BF16;
    switch (L) {
#define HY_BW(LM) \
    case 1 << LM: return bf ? launch_bw_t<LM, __nv_bfloat16>(p, s) : launch_bw_t<LM, float>(p, s);
        HY_BW(9) HY_BW(10) HY_BW(11) HY_BW(12) HY_BW(13)
#undef HY_BW
        default: return set_error(HY_ERR_UNSUPPORTED, "fused backward: L=%d not built", L);
    }
}

}  // namespace hy
