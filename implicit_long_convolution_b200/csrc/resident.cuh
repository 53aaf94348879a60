// resident.cuh -- single-launch FFT convolution with gating, one sequence row
// per CTA held on chip (registers + shared memory) across all orders.
//
// Per row (a real sequence of L samples, transform length n = 2M):
//   pack      z[m] = s[2m] + i s[2m+1], m < M (rows zero-padded to n)
//   forward   Z = FFT_M(z)                       (block_fft, registers + smem)
//   split     X[k] = ½(Z[k] + Z*[M-k]) - ½ i W_n^k (Z[k] - Z*[M-k]),  k = 0..M
//   multiply  Y[k] = X[k] · H[k]                 (filter spectrum or gate)
//   merge     Z'[k] = (Y[k] + Y*[M-k]) + i W_n^{-k} (Y[k] - Y*[M-k])
//   inverse   z' = IFFT_M(Z') / n ;  c[2m] = Re z'[m], c[2m+1] = Im z'[m]
//   epilogue  z_k = x_k ⊙ c                    (next order starts from z_k)
// The skip term D_k·z_{k-1} is applied in the spectrum (bins times H + D_k).
// Split and merge of bins k and M-k are done together by the thread owning
// k < M/2; the partner value crosses shared memory.  Only the first L
// samples of each order are kept (the rest of the padded row restarts at 0),
// which makes every order a linear, causal convolution.  In the circular
// variant (spectral gate) n = L and nothing is padded.
#pragma once
#include "bulk_copy.cuh"
#include "fft_core.cuh"

namespace hy {

constexpr int kMaxOrders = 8;   // filters per operator call (order <= 9)


__host__ __device__ constexpr int resident_log_p(int log_m) {
    return log_m - 5 < 2 ? 2 : (log_m - 5 > 5 ? 5 : log_m - 5);
}

struct ResidentParams {
    int64_t n_rows;
    int L;                       // valid samples per row
    int K;                       // orders (filters) chained in this launch
    int B, D;                    // CTA c -> row (c % B) * D + c / B when remap
    int remap;
    const void *u;               // z_0 rows (IO dtype), row stride L
    const void *gate[kMaxOrders];
    const float2 *spec[kMaxOrders];
    const float *skip[kMaxOrders];
    int64_t spec_row_stride;     // complex elements between spectrum rows
    int64_t sdiv, smod;          // spectrum channel of row r: (r / sdiv) % smod
    int64_t spec_batch_stride;   // per sample r / (sdiv * smod); 0 = shared
    void *y;
    float scale;                 // 1 / (2n): folds the halving of split and the 1/n
    const float2 *tw_fft;
    const float2 *tw_split;
    uint32_t *fault;             // device fault word (bounded waits), or NULL
};

// The skip term folds into the spectrum: h * u + D u = (h + D delta) * u, and
// the spectrum of delta is 1 at every bin, so each bin is multiplied by H + D.
// Bins k = t + m*T (m < P/2) pair with M - k; a batch of pairs issues its
// spectrum loads together so their L2 round trips overlap.  The split twiddle
// W_n^k (n = 2M) is W_n^t * W_{2P}^m: one table entry per thread times a
// compile-time rotation.
template <int LOG_M, int LOG_P>
__device__ __forceinline__ void split_multiply_merge(float2 (&x)[1 << LOG_P], float2 *sbuf, int t,
                                                     const float2 *__restrict__ H,
                                                     const float2 *__restrict__ tws, float dk) {
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int BATCH = (P / 2) < 4 ? (P / 2) : 4;
    store_own<LOG_M, LOG_P>(x, sbuf, t);
    const float2 wt0 = ldc(tws + t);
    __syncthreads();
    auto batch = [&](auto bc) {
        constexpr int m0 = decltype(bc)::value * BATCH;
        float2 hk[BATCH], hn[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            const int k = t + (m0 + j) * T;
            hk[j] = ldv(H + k);
            hn[j] = ldv(H + (M - k));
            hk[j].x += dk;
            hn[j].x += dk;
        }
        auto pair = [&](auto jc) {
            constexpr int j = decltype(jc)::value;
            constexpr int m = m0 + j;
            const int k = t + m * T;
            if (k == 0) {
                // DC and Nyquist: X[0] = Re Z0 + Im Z0, X[M] = Re Z0 - Im Z0
                // (both real, doubled here); only the real part of the product
                // is kept.  H[M] = hn[j] at k = 0.
                const float2 z0 = x[0];
                const float y0 = 2.f * (z0.x + z0.y) * hk[j].x;
                const float yM = 2.f * (z0.x - z0.y) * hn[j].x;
                x[0] = make_float2(y0 + yM, y0 - yM);
            } else {
                const float2 zk = x[m];
                const float2 zn = sbuf[partner_slot<LOG_M, LOG_P>(t, m)];
                const float2 A = make_float2(zk.x + zn.x, zk.y - zn.y);   // Z[k] + Z*[M-k]
                const float2 Bv = make_float2(zk.x - zn.x, zk.y + zn.y);  // Z[k] - Z*[M-k]
                const float2 w = rot<-1, 2 * P, m>(wt0);                  // W_n^k
                const float2 wB = cmul(Bv, w);
                const float2 C = make_float2(wB.y, -wB.x);                // -i W B
                const float2 Xk = cadd(A, C);                             // 2 X[k]
                const float2 Xn = cconj(csub(A, C));                      // 2 X[M-k]
                const float2 Yk = cmul(Xk, hk[j]);
                const float2 Yn = cmul(Xn, hn[j]);
                const float2 A2 = make_float2(Yk.x + Yn.x, Yk.y - Yn.y);
                const float2 B2 = make_float2(Yk.x - Yn.x, Yk.y + Yn.y);
                const float2 cB = cmulc(B2, w);
                const float2 C2 = make_float2(-cB.y, cB.x);               // i W^-1 B'
                x[m] = cadd(A2, C2);
                sbuf[partner_slot<LOG_M, LOG_P>(t, m)] = cconj(csub(A2, C2));
            }
        };
        fold_seq(pair, std::make_integer_sequence<int, BATCH>{});
    };
    fold_seq(batch, std::make_integer_sequence<int, (P / 2) / BATCH>{});
    if (t == 0) {
        // k = M/2 pairs with itself: Z'[M/2] = 4 Z[M/2] conj(H[M/2] + D) (doubled scale)
        const float2 z = x[P / 2];
        float2 hm = ldv(H + M / 2);
        hm.x += dk;
        const float2 r = cmulc(z, hm);
        x[P / 2] = make_float2(4.f * r.x, 4.f * r.y);
    }
    __syncthreads();
#pragma unroll
    for (int m = P / 2; m < P; ++m)
        if (!(t == 0 && m == P / 2)) x[m] = sbuf[own_slot<LOG_M, LOG_P>(t, m)];
    __syncthreads();
}

// CTAs per SM the register budget is sized for (128 registers per thread at
// 256 threads): two CTAs overlap one's barriers with the other's arithmetic.
__host__ __device__ constexpr int resident_min_blocks(int log_m) {
    return ((1 << log_m) >> resident_log_p(log_m)) <= 256 ? 2 : 1;
}

// CHAIN = false: exactly one order (K = 1): order-2 operator, single gated
// convolution, spectral gate.  CHAIN = true: K >= 1 orders in a runtime loop
// (the loop costs registers, so the single-order case has its own build).
template <int LOG_M, typename IO, bool CIRC, bool CHAIN>
__global__ void __launch_bounds__((1 << LOG_M) >> resident_log_p(LOG_M), resident_min_blocks(LOG_M))
resident_conv_kernel(const ResidentParams p) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int PIN = CIRC ? P : P / 2;   // registers carrying samples
    using IOT = IOTraits<IO>;

    extern __shared__ float2 smem[];
    float2 *sbuf = smem;

    const int t = threadIdx.x;
    const int64_t c = blockIdx.x;
    const int64_t row = p.remap ? (c % p.B) * (int64_t)p.D + c / p.B : c;
    const int64_t ch = (row / p.sdiv) % p.smod;
    const int64_t smp = row / (p.sdiv * p.smod);
    const int L = p.L;
    const bool pairs = (L & 1) == 0;
    const IO *u = reinterpret_cast<const IO *>(p.u) + row * (int64_t)L;

    float2 x[P];
#pragma unroll
    for (int m = 0; m < P; ++m) {
        x[m] = make_float2(0.f, 0.f);
        if (m < PIN) {
            const int i0 = 2 * (t + m * T);
            if (pairs) {
                if (i0 < L) x[m] = IOT::load2(u + i0);
            } else {
                if (i0 < L) x[m].x = IOT::load(u + i0);
                if (i0 + 1 < L) x[m].y = IOT::load(u + i0 + 1);
            }
        }
    }

    auto one_order = [&](const int k, const bool last) {
        // thread index re-read per order (volatile): addresses derived from it
        // are formed inside the order loop instead of held across it
        int t;
        asm volatile("mov.u32 %0, %%tid.x;" : "=r"(t));
        block_fft<LOG_M, LOG_P, -1, !CIRC>(x, sbuf, t, p.tw_fft);
        const float dk = p.skip[k] ? ldv(p.skip[k] + ch) : 0.f;
        const float2 *H = p.spec[k] + smp * p.spec_batch_stride + ch * p.spec_row_stride;
        split_multiply_merge<LOG_M, LOG_P>(x, sbuf, t, H, p.tw_split, dk);
        block_fft<LOG_M, LOG_P, +1, false>(x, sbuf, t, p.tw_fft);

        const IO *g = reinterpret_cast<const IO *>(p.gate[k]);
        const IO *grow = g ? g + row * (int64_t)L : nullptr;
        IO *yout = reinterpret_cast<IO *>(p.y) + row * (int64_t)L;
        // batches of EB samples: issue the batch's gate loads first (the
        // output stores would otherwise order each load behind them)
        constexpr int EB = (PIN < 8) ? PIN : 8;
#pragma unroll
        for (int m0 = 0; m0 < PIN; m0 += EB) {
            float2 gv[EB];
#pragma unroll
            for (int j = 0; j < EB; ++j) {
                const int i0 = 2 * (t + (m0 + j) * T);
                gv[j] = make_float2(1.f, 1.f);
                if (grow) {
                    if (pairs) {
                        if (i0 < L) gv[j] = IOT::load2(grow + i0);
                    } else {
                        if (i0 < L) gv[j].x = IOT::load(grow + i0);
                        if (i0 + 1 < L) gv[j].y = IOT::load(grow + i0 + 1);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < EB; ++j) {
                const int m = m0 + j;
                const int i0 = 2 * (t + m * T);
                float2 z = make_float2(x[m].x * p.scale * gv[j].x, x[m].y * p.scale * gv[j].y);
                if (i0 >= L) z.x = 0.f;
                if (i0 + 1 >= L) z.y = 0.f;
                if (last) {
                    if (pairs) {
                        if (i0 < L) IOT::store2(yout + i0, z);
                    } else {
                        if (i0 < L) IOT::store(yout + i0, z.x);
                        if (i0 + 1 < L) IOT::store(yout + i0 + 1, z.y);
                    }
                } else {
                    x[m] = z;
                }
            }
        }
#pragma unroll
        for (int m = PIN; m < P; ++m) x[m] = make_float2(0.f, 0.f);
    };

    if constexpr (CHAIN) {
        for (int k = 0; k < p.K; ++k) one_order(k, k == p.K - 1);
    } else {
        one_order(0, true);
    }
}

// ----------------------------------------------------------------------------
// Streaming variant for one order (K = 1) with L = 2^LOG_M (causal) or
// L = 2^(LOG_M+1) (circular) samples per row: a persistent CTA walks its rows
// and overlaps HBM with the FFTs.  While row r is being transformed, TMA bulk
// copies bring row r+1's input and row r's gate into shared memory (stage
// buffers next to the FFT exchange buffer), each landing on its own mbarrier;
// the skip term rides on the spectrum (see split_multiply_merge).  Without
// PF_GATE (when two stage buffers would not fit) the gate is read from
// global memory in the epilogue (an L2 bulk prefetch of the gate row at the
// start of the row was measured slower at the 16384-point spectral gate).  Every wait is bounded: a copy that has not
// landed within the limit records a fault bit, and the CTA stops at the next
// row boundary (after waiting, again bounded, for its copies in flight).
// ----------------------------------------------------------------------------

// float2 slots before the stage buffers (even, so they start 16-byte aligned)
__host__ __device__ constexpr int stream_stage_offset(int m) { return ((spad_size(m) + 1) / 2) * 2; }
// dynamic shared memory of the streaming kernel
__host__ __device__ constexpr size_t stream_smem_bytes(int log_m, int io_bytes, bool circ, bool pf_gate) {
    return (size_t)stream_stage_offset(1 << log_m) * 8 +
           (size_t)(circ ? 2 : 1) * (1 << log_m) * io_bytes * (pf_gate ? 2 : 1);
}
// prefetch the gate too when both stage buffers fit beside the CTAs per SM the
// registers allow (about 113 KB each for two CTAs, 227 KB for one)
__host__ __device__ constexpr bool stream_pf_gate(int log_m, int io_bytes, bool circ) {
    return stream_smem_bytes(log_m, io_bytes, circ, true) <=
           (resident_min_blocks(log_m) >= 2 ? (size_t)113 * 1024 : (size_t)227 * 1024);
}

template <int LOG_M, typename IO, bool CIRC, bool PF_GATE>
__global__ void __launch_bounds__((1 << LOG_M) >> resident_log_p(LOG_M), resident_min_blocks(LOG_M))
resident_stream_kernel(const ResidentParams p) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int PIN = CIRC ? P : P / 2;
    constexpr int L = CIRC ? 2 * M : M;                  // samples per row
    constexpr uint32_t ROW_BYTES = (uint32_t)(L * sizeof(IO));
    static_assert(ROW_BYTES % 16 == 0 && ROW_BYTES < (1u << 20), "bulk copy size");
    using IOT = IOTraits<IO>;

    extern __shared__ __align__(128) float2 smem[];   // stage buffers take 16-byte aligned bulk copies
    float2 *sbuf = smem;
    IO *in_st = reinterpret_cast<IO *>(smem + stream_stage_offset(M));   // 16-byte aligned
    IO *g_st = in_st + L;
    __shared__ uint64_t bars[2];                         // [0]: input stage, [1]: gate stage
    __shared__ int s_abort;

    const IO *ubase = reinterpret_cast<const IO *>(p.u);
    const IO *gbase = reinterpret_cast<const IO *>(p.gate[0]);
    IO *ybase = reinterpret_cast<IO *>(p.y);
    const bool gate_pf = PF_GATE && gbase != nullptr;
    auto row_of = [&](int64_t c) { return p.remap ? (c % p.B) * (int64_t)p.D + c / p.B : c; };

    int64_t c = blockIdx.x;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init_fence();
        s_abort = 0;
    }
    __syncthreads();
    if (threadIdx.x == 0 && c < p.n_rows) bulk_g2s(in_st, ubase + row_of(c) * L, ROW_BYTES, &bars[0]);
    // waits taken on each barrier; every copy issued is waited on by the
    // iteration that issued it (gate) or the next one (input), so at any
    // exit of the loop these are also the copies issued
    uint32_t w_in = 0, w_g = 0;
    for (; c < p.n_rows; c += gridDim.x) {
        // the thread index re-read per row (volatile) so the addresses derived
        // from it are formed inside the loop instead of held across it
        int t;
        asm volatile("mov.u32 %0, %%tid.x;" : "=r"(t));
        const int64_t row = row_of(c);
        const int64_t ch = (row / p.sdiv) % p.smod;
        const int64_t smp = row / (p.sdiv * p.smod);
        if (!mbar_wait(&bars[0], w_in & 1)) {
            record_fault(p.fault, HY_FAULT_STREAM_INPUT);
            s_abort = 1;
        }
        ++w_in;
        float2 x[P];
#pragma unroll
        for (int m = 0; m < P; ++m) {
            x[m] = make_float2(0.f, 0.f);
            if (m < PIN) {
                const int i0 = 2 * (t + m * T);
                if constexpr (sizeof(IO) == 2) {
                    const uint32_t b = *reinterpret_cast<const uint32_t *>(in_st + i0);
                    x[m] = make_float2(__uint_as_float(b << 16), __uint_as_float(b & 0xffff0000u));
                } else {
                    x[m] = *reinterpret_cast<const float2 *>(in_st + i0);
                }
            }
        }
        __syncthreads();                                  // stage buffers free for the next copies
        if (s_abort) break;                               // uniform: read between two barriers
        if (t == 0) {
            fence_proxy_async_smem();
            if (gate_pf) bulk_g2s(g_st, gbase + row * L, ROW_BYTES, &bars[1]);
            if (c + gridDim.x < p.n_rows) bulk_g2s(in_st, ubase + row_of(c + gridDim.x) * L, ROW_BYTES, &bars[0]);
        }

        block_fft<LOG_M, LOG_P, -1, !CIRC>(x, sbuf, t, p.tw_fft);
        const float dk = p.skip[0] ? ldv(p.skip[0] + ch) : 0.f;
        const float2 *H = p.spec[0] + smp * p.spec_batch_stride + ch * p.spec_row_stride;
        split_multiply_merge<LOG_M, LOG_P>(x, sbuf, t, H, p.tw_split, dk);
        block_fft<LOG_M, LOG_P, +1, false>(x, sbuf, t, p.tw_fft);

        if (gate_pf) {
            if (!mbar_wait(&bars[1], w_g & 1)) {          // the gate of this row has landed
                record_fault(p.fault, HY_FAULT_STREAM_GATE);
                s_abort = 1;                              // seen after the next row's first barrier
            }
            ++w_g;
        }
        IO *yout = ybase + row * (int64_t)L;
#pragma unroll
        for (int m = 0; m < PIN; ++m) {
            const int i0 = 2 * (t + m * T);
            float2 z = make_float2(x[m].x * p.scale, x[m].y * p.scale);
            if (gbase) {
                float2 gv;
                if (gate_pf) {
                    if constexpr (sizeof(IO) == 2) {
                        const uint32_t b = *reinterpret_cast<const uint32_t *>(g_st + i0);
                        gv = make_float2(__uint_as_float(b << 16), __uint_as_float(b & 0xffff0000u));
                    } else {
                        gv = *reinterpret_cast<const float2 *>(g_st + i0);
                    }
                } else {
                    gv = IOT::load2(gbase + row * (int64_t)L + i0);
                }
                z = make_float2(z.x * gv.x, z.y * gv.y);
            }
            IOT::store2(yout + i0, z);
        }
    }
    // no copy may still be landing in shared memory when the CTA exits
    if (threadIdx.x == 0) {
        if (w_in && !mbar_wait(&bars[0], (w_in - 1) & 1)) record_fault(p.fault, HY_FAULT_STREAM_INPUT);
        if (w_g && !mbar_wait(&bars[1], (w_g - 1) & 1)) record_fault(p.fault, HY_FAULT_STREAM_GATE);
    }
}

// Filter spectrum rows: H[r, k] = Σ_t h[r, t] W_n^{kt}, k = 0..M, for rows of
// L fp32 samples (zero-padded to n = 2M, or exactly n = L when circular).
template <int LOG_M, bool CIRC>
__global__ void __launch_bounds__((1 << LOG_M) >> resident_log_p(LOG_M))
spectrum_rows_kernel(int64_t n_rows, int L, const float *__restrict__ h, float2 *__restrict__ Hout,
                     const float2 *__restrict__ tw_fft, const float2 *__restrict__ tws) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int PIN = CIRC ? P : P / 2;
    extern __shared__ float2 smem[];
    float2 *sbuf = smem;
    const int t = threadIdx.x;
    const int64_t row = blockIdx.x;
    const float *hr = h + row * (int64_t)L;
    float2 *Hr = Hout + row * (int64_t)(M + 1);
    const bool pairs = (L & 1) == 0;

    float2 x[P];
#pragma unroll
    for (int m = 0; m < P; ++m) {
        x[m] = make_float2(0.f, 0.f);
        if (m < PIN) {
            const int i0 = 2 * (t + m * T);
            if (pairs) {
                if (i0 < L) x[m] = __ldg(reinterpret_cast<const float2 *>(hr + i0));
            } else {
                if (i0 < L) x[m].x = __ldg(hr + i0);
                if (i0 + 1 < L) x[m].y = __ldg(hr + i0 + 1);
            }
        }
    }
    block_fft<LOG_M, LOG_P, -1, !CIRC>(x, sbuf, t, tw_fft);
    store_own<LOG_M, LOG_P>(x, sbuf, t);
    __syncthreads();
#pragma unroll
    for (int m = 0; m < P / 2; ++m) {
        const int k = t + m * T;
        if (k == 0) {
            const float2 z0 = x[0];
            Hr[0] = make_float2(z0.x + z0.y, 0.f);
            Hr[M] = make_float2(z0.x - z0.y, 0.f);
        } else {
            const float2 zk = x[m];
            const float2 zn = sbuf[partner_slot<LOG_M, LOG_P>(t, m)];
            const float2 A = make_float2(zk.x + zn.x, zk.y - zn.y);
            const float2 Bv = make_float2(zk.x - zn.x, zk.y + zn.y);
            const float2 wB = cmul(Bv, __ldg(tws + k));
            const float2 C = make_float2(wB.y, -wB.x);
            const float2 Xk = cadd(A, C);
            const float2 Xn = cconj(csub(A, C));
            Hr[k] = make_float2(0.5f * Xk.x, 0.5f * Xk.y);
            Hr[M - k] = make_float2(0.5f * Xn.x, 0.5f * Xn.y);
        }
    }
    if (t == 0) Hr[M / 2] = cconj(x[P / 2]);
}

}  // namespace hy
