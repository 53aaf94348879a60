// fft_core.cuh -- register/shared-memory FFT building blocks for sm_100a.
//
// A complex FFT of size M is computed by T = M / P cooperating threads; thread
// t owns the P elements t + T*m (m = 0..P-1) in registers.  The transform is a
// self-sorting (Stockham) sequence of radix-R stages.  Stage s with radix R and
// p = product of the earlier radices takes butterfly i = t + q*T, reads its
// inputs x_r = in[i + r*M/R] -- always the thread's own registers q + r*P/R --
// multiplies x_r by W_{pR}^{k r} (k = i mod p), does a radix-R DFT in
// registers and writes output r to (i - k)*R + k + r*p.  Between stages the
// outputs go through shared memory; the last stage's outputs land exactly in
// the thread's own slots, so a size-M FFT needs (stages - 1) exchanges and
// leaves natural-order results in registers.
//
// The radix-R DFT is a decimation-in-frequency network fully unrolled at
// compile time; its internal twiddles are compile-time constants and trivial
// ones (±1, ±i, (±1±i)/√2) cost no multiply.
#pragma once
#include "common.cuh"

namespace hy {

// ----------------------------------------------------------------------------
// Radix-R DFT (R = 2^p <= 64) in registers, DIF, bit-reversed output:
// after dft_dif<R>(a), a[j] holds X[bitrev_R(j)].
// ----------------------------------------------------------------------------
template <int DIR, int SPAN, int J>
__device__ __forceinline__ void bfly_dif(float2 &u, float2 &v) {
    float2 s = cadd(u, v);
    float2 d = csub(u, v);
    u = s;
    v = rot<DIR, 2 * SPAN, J>(d);
}

template <int DIR, int SPAN, int... J>
__device__ __forceinline__ void dif_block(float2 *a, std::integer_sequence<int, J...>) {
    (bfly_dif<DIR, SPAN, J>(a[J], a[J + SPAN]), ...);
}

// first layer when the upper half of the inputs is known to be zero:
// (u, 0) -> (u, u * W)
template <int DIR, int SPAN, int J>
__device__ __forceinline__ void bfly_dif_zero(float2 &u, float2 &v) {
    v = rot<DIR, 2 * SPAN, J>(u);
}
template <int DIR, int SPAN, int... J>
__device__ __forceinline__ void dif_block_zero(float2 *a, std::integer_sequence<int, J...>) {
    (bfly_dif_zero<DIR, SPAN, J>(a[J], a[J + SPAN]), ...);
}

template <int R, int DIR, int SPAN>
__device__ __forceinline__ void dif_layers(float2 *a) {
#pragma unroll
    for (int start = 0; start < R; start += 2 * SPAN)
        dif_block<DIR, SPAN>(a + start, std::make_integer_sequence<int, SPAN>{});
    if constexpr (SPAN > 1) dif_layers<R, DIR, SPAN / 2>(a);
}

template <int R, int DIR, bool UPPER_ZERO = false>
__device__ __forceinline__ void dft_dif(float2 *a) {
    static_assert(R >= 1 && (R & (R - 1)) == 0, "radix must be a power of two");
    if constexpr (R == 1) {
        return;
    } else if constexpr (UPPER_ZERO) {
        dif_block_zero<DIR, R / 2>(a, std::make_integer_sequence<int, R / 2>{});
        if constexpr (R > 2) dif_layers<R, DIR, R / 4>(a);
    } else {
        dif_layers<R, DIR, R / 2>(a);
    }
}

__host__ __device__ constexpr int ct_log2(int x) { return x <= 1 ? 0 : 1 + ct_log2(x >> 1); }
__host__ __device__ constexpr int bitrev(int j, int bits) {
    int r = 0;
    for (int b = 0; b < bits; ++b) r |= ((j >> b) & 1) << (bits - 1 - b);
    return r;
}

// ----------------------------------------------------------------------------
// Radix plan: radix P while it fits, then the remainder (e.g. 8192 points with
// 32 per thread: 32 x 32 x 8).  Stage 0 needs no twiddles.  (A balanced plan,
// 32 x 16 x 16, has two butterflies per thread in the twiddled stages and
// needs more registers for the same instruction count.)  Shared by the device
// code and the host-side twiddle-table builder.
// ----------------------------------------------------------------------------
__host__ __device__ constexpr int plan_stages(int log_m, int log_p) {
    return (log_m + log_p - 1) / log_p;
}
__host__ __device__ constexpr int plan_log_radix(int log_m, int log_p, int s) {
    return (s < plan_stages(log_m, log_p) - 1) ? log_p : (log_m - log_p * (plan_stages(log_m, log_p) - 1));
}
__host__ __device__ constexpr int plan_log_p(int log_m, int log_p, int s) {
    int acc = 0;
    for (int i = 0; i < s; ++i) acc += plan_log_radix(log_m, log_p, i);
    return acc;
}
// Columns of stage s's twiddle table.  Butterfly i = t + q*T of a stage with
// p = 2^plan_log_p needs W_{pR}^{(i mod p) r}.  When p <= T that is the same
// for every q (column i mod p).  When p > T (only the last stage, where
// i < p) W^{(t + qT) r} = W^{t r} * W^{qT r}: the table keeps the T columns
// W^{t r} and the second factor is a compile-time constant.
__host__ __device__ constexpr int plan_tw_cols(int log_m, int log_p, int s) {
    return (1 << plan_log_p(log_m, log_p, s)) < (1 << (log_m - log_p)) ? (1 << plan_log_p(log_m, log_p, s))
                                                                         : (1 << (log_m - log_p));
}
// twiddle entries of stage s: (R - 1) * columns (none for stage 0)
__host__ __device__ constexpr int plan_tw_count(int log_m, int log_p, int s) {
    return s == 0 ? 0 : ((1 << plan_log_radix(log_m, log_p, s)) - 1) * plan_tw_cols(log_m, log_p, s);
}
__host__ __device__ constexpr int plan_tw_offset(int log_m, int log_p, int s) {
    int acc = 0;
    for (int i = 0; i < s; ++i) acc += plan_tw_count(log_m, log_p, i);
    return acc;
}
__host__ __device__ constexpr int plan_tw_total(int log_m, int log_p) {
    return plan_tw_offset(log_m, log_p, plan_stages(log_m, log_p));
}

// Shared-memory slot of complex element e: one pad slot every 2^SH elements
// keeps the stride-R writes of the first stage conflict-free.  SH = 5 (a pad
// every 32) is the default of the row kernels, whose FFTs span whole warps;
// FFTs of 8 or 16 threads (several per warp) take SH = 3 or 4.
template <int SH>
__device__ __forceinline__ int spadx(int e) { return e + (e >> SH); }
__device__ __forceinline__ int spad(int e) { return spadx<5>(e); }
__host__ __device__ constexpr int spad_size(int m) { return m + (m >> 5) + 1; }

// x[m] = element t + m*T of a padded shared buffer (linear addressing when
// T is a multiple of 2^SH).
template <int LOG_M, int LOG_P, int SH = 5>
__device__ __forceinline__ void load_own(float2 (&x)[1 << LOG_P], const float2 *sbuf, int t) {
    constexpr int P = 1 << LOG_P;
    constexpr int T = (1 << LOG_M) / P;
    if constexpr (T % (1 << SH) == 0) {
        const float2 *src = sbuf + spadx<SH>(t);
        constexpr int STEP = T + (T >> SH);
#pragma unroll
        for (int m = 0; m < P; ++m) x[m] = src[m * STEP];
    } else {
#pragma unroll
        for (int m = 0; m < P; ++m) x[m] = sbuf[spadx<SH>(t + m * T)];
    }
}
template <int LOG_M, int LOG_P, int SH = 5>
__device__ __forceinline__ void store_own(const float2 (&x)[1 << LOG_P], float2 *sbuf, int t) {
    constexpr int P = 1 << LOG_P;
    constexpr int T = (1 << LOG_M) / P;
    if constexpr (T % (1 << SH) == 0) {
        float2 *dst = sbuf + spadx<SH>(t);
        constexpr int STEP = T + (T >> SH);
#pragma unroll
        for (int m = 0; m < P; ++m) dst[m * STEP] = x[m];
    } else {
#pragma unroll
        for (int m = 0; m < P; ++m) sbuf[spadx<SH>(t + m * T)] = x[m];
    }
}
// Padded slot of the thread's own element t + m*T.
template <int LOG_M, int LOG_P>
__device__ __forceinline__ int own_slot(int t, int m) {
    constexpr int T = (1 << LOG_M) >> LOG_P;
    if constexpr (T % 32 == 0) return spad(t) + m * (T + T / 32);
    else return spad(t + m * T);
}
// Address of padded element M - (t + m*T) for m = 0: the partner bins of the
// real-FFT split walk down from here in steps of -(T + T/32).
template <int LOG_M, int LOG_P>
__device__ __forceinline__ int partner_slot(int t, int m) {
    constexpr int M = 1 << LOG_M;
    constexpr int T = M >> LOG_P;
    if constexpr (T % 32 == 0) return spad(M - t) - m * (T + T / 32);
    else return spad(M - t - m * T);
}

// Synchronisation of the threads that share one FFT.
struct SyncBlock {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct SyncWarp {
    __device__ __forceinline__ void operator()() const { __syncwarp(); }
};

// Butterfly Q of a wide last stage: y[r] = x[Q + r*NB] times the twiddle
// wb[r] * W_N^{QT r} (forward; conjugated for DIR = +1), then the radix-R DFT.
// QT = Q*T is a template constant, so W_N^{QT r} is a compile-time rotation
// (free for Q = 0).
template <int DIR, int N, int QT, int... J>
__device__ __forceinline__ void tw_apply_q(float2 *y, const float2 *wb, std::integer_sequence<int, J...>) {
    ((y[J + 1] = cmul_dir<DIR>(y[J + 1], rot<-1, N, QT * (J + 1)>(wb[J + 1]))), ...);
}
template <int R, int NB, int T, int N, int DIR, bool UPPER_ZERO, int P, int... Q>
__device__ __forceinline__ void wide_last_stage(float2 (&x)[P], float2 (&y)[NB][R], const float2 *wb,
                                                std::integer_sequence<int, Q...>) {
    auto one = [&](auto qc) {
        constexpr int q = decltype(qc)::value;
#pragma unroll
        for (int r = 0; r < R; ++r) y[q][r] = x[q + r * NB];
        tw_apply_q<DIR, N, q * T>(y[q], wb, std::make_integer_sequence<int, R - 1>{});
        dft_dif<R, DIR, UPPER_ZERO>(y[q]);
    };
    (one(std::integral_constant<int, Q>{}), ...);
}

// ----------------------------------------------------------------------------
// One Stockham stage.  x: the thread's P registers.  If LAST, outputs are left
// in registers (natural order); otherwise written to sbuf and read back.
// tw: this stage's table, layout [(r-1) * p + k] = W_{pR}^{k r} (forward).
// ----------------------------------------------------------------------------
template <int LOG_M, int LOG_P, int S, int DIR, bool UPPER_ZERO, typename Sync, int SH = 5>
__device__ __forceinline__ void fft_stage(float2 (&x)[1 << LOG_P], float2 *sbuf, int t,
                                          const float2 *__restrict__ tw, Sync sync) {
    constexpr int M = 1 << LOG_M;
    constexpr int P = 1 << LOG_P;
    constexpr int T = M / P;
    constexpr int LR = plan_log_radix(LOG_M, LOG_P, S);
    constexpr int R = 1 << LR;
    constexpr int LPS = plan_log_p(LOG_M, LOG_P, S);
    constexpr int PS = 1 << LPS;
    constexpr int NB = P / R;                  // butterflies per thread
    constexpr bool LAST = (S == plan_stages(LOG_M, LOG_P) - 1);

    float2 y[NB][R];
    if constexpr (S > 0 && PS > T) {
        static_assert(LAST, "a stage wider than the thread count must be the last");
        // W^{(t + qT) r} = W^{t r} * W^{qT r}; the second factor is constant
        float2 wb[R];
#pragma unroll
        for (int r = 1; r < R; ++r) wb[r] = __ldg(tw + (r - 1) * T + t);
        wide_last_stage<R, NB, T, PS * R, DIR, UPPER_ZERO>(x, y, wb, std::make_integer_sequence<int, NB>{});
    } else {
#pragma unroll
    for (int q = 0; q < NB; ++q) {
        const int i = t + q * T;
        const int k = i & (PS - 1);
#pragma unroll
        for (int r = 0; r < R; ++r) y[q][r] = x[q + r * NB];
        if constexpr (S > 0) {
#pragma unroll
            for (int r = 1; r < R; ++r) y[q][r] = cmul_dir<DIR>(y[q][r], __ldg(tw + (r - 1) * PS + k));
        }
        dft_dif<R, DIR, UPPER_ZERO>(y[q]);
    }
    }
    if constexpr (LAST) {
#pragma unroll
        for (int q = 0; q < NB; ++q)
#pragma unroll
            for (int r = 0; r < R; ++r) x[q + r * NB] = y[q][bitrev(r, LR)];
    } else {
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int i = t + q * T;
            const int k = i & (PS - 1);
            const int base = (i - k) * R + k;
            if constexpr (PS % (1 << SH) == 0 || (PS == 1 && R <= (1 << SH))) {
                // padded address is linear in r here: one base, constant steps
                float2 *dst = sbuf + spadx<SH>(base);
                constexpr int STEP = PS + (PS >> SH);
#pragma unroll
                for (int r = 0; r < R; ++r) dst[r * STEP] = y[q][bitrev(r, LR)];
            } else {
#pragma unroll
                for (int r = 0; r < R; ++r) sbuf[spadx<SH>(base + r * PS)] = y[q][bitrev(r, LR)];
            }
        }
        sync();
        load_own<LOG_M, LOG_P, SH>(x, sbuf, t);
        sync();
    }
}

template <int LOG_M, int LOG_P, int S, int DIR, bool UPPER_ZERO, typename Sync, int SH>
__device__ __forceinline__ void fft_stages_from(float2 (&x)[1 << LOG_P], float2 *sbuf, int t,
                                                const float2 *__restrict__ tw, Sync sync) {
    constexpr int NS = plan_stages(LOG_M, LOG_P);
    if constexpr (S < NS) {
        fft_stage<LOG_M, LOG_P, S, DIR, (S == 0) && UPPER_ZERO, Sync, SH>(x, sbuf, t,
                                                                           tw + plan_tw_offset(LOG_M, LOG_P, S), sync);
        fft_stages_from<LOG_M, LOG_P, S + 1, DIR, UPPER_ZERO, Sync, SH>(x, sbuf, t, tw, sync);
    }
}

// Full complex FFT of size 2^LOG_M (unnormalised).  DIR = -1: forward
// (e^{-2πi/M}); +1: inverse.  UPPER_ZERO: elements M/2..M-1 of the input are
// zero (zero-padded rows) and are not read.  SH: the padding of sbuf (spadx).
template <int LOG_M, int LOG_P, int DIR, bool UPPER_ZERO = false, typename Sync = SyncBlock, int SH = 5>
__device__ __forceinline__ void block_fft(float2 (&x)[1 << LOG_P], float2 *sbuf, int t,
                                          const float2 *__restrict__ tw, Sync sync = Sync{}) {
    fft_stages_from<LOG_M, LOG_P, 0, DIR, UPPER_ZERO, Sync, SH>(x, sbuf, t, tw, sync);
}

}  // namespace hy
