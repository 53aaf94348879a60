// resident_tc.cu -- the streaming FFT convolution of one order with the two
// radix-32 stages of each FFT done as DFT matrix products on the tcgen05
// tensor cores: rows of L = 8192 bf16 samples (M = 8192 complex points, the
// order-2 operator at its ~153M-model width and 8K length), causal.
//
// The transform plan is the on-chip kernel's (resident.cuh): Stockham stages
// of radix 32, 32 and 8 over M = 8192, 256 threads, thread t owning elements
// t + 256 m.  In a radix-32 stage every thread holds the 32 inputs of one
// butterfly, so the 256 butterflies of a stage are one matrix product
//   D[t, r'] = Σ_r A[t, r] · F[r, r'],   F[r, r'] = W_32^{± r r'},
// on 2 M-tiles of 128 rows.  Complex values are carried as real K-blocks:
// A row t = [Re a_t[0..31] | Im a_t[0..31]] (64 K elements), the constant
// operand row r' = [cos(2π r r'/32) | sin(2π r r'/32)] (r = 0..31), and
//   forward:  Re D = Re a·C + Im a·S,   Im D = Im a·C − Re a·S
//   inverse:  Re D = Re a·C − Im a·S,   Im D = Im a·C + Re a·S
// as four K=16 MMAs per part (M = 128, N = 32), the minus signs through the
// instruction's negate-B bit.  The accumulators live in TMEM (Re at columns
// 64 i, Im at 64 i + 32 for M-tile i); thread t reads its own row back with
// tcgen05.ld (warp w reads lanes 32 (w % 4) .. + 31 of tile w / 4).
//
// Precision: every fp32 operand x is split into bf16 parts hi = rn(x),
// lo = rn(x − hi), and products are summed as hi·hi + hi·lo + lo·hi with
// fp32 accumulation (relative error of each product about 2^-17; the
// dropped lo·lo term is smaller).  The first forward stage takes the bf16
// input samples themselves, which are exact, so it needs only hi·(F_hi +
// F_lo).  The radix-8 stage, the twiddles, the real-FFT split / merge with
// the spectrum product (and skip term), the gate and the bf16 rounding of
// the output are the fp32 SIMT code of resident.cuh.  Zero-padded halves
// are skipped as there: the first forward stage multiplies only the 16
// non-zero inputs of each butterfly (K = 16 + 16 instead of 64).
//
// The A operand of a stage (256 rows x 128 bytes, hi and lo = 64 KB,
// K-major, 128-byte swizzle) occupies the bytes of the shared exchange
// buffer, which is free while the MMAs run.  Rows are staged by TMA bulk
// copies on mbarriers as in the streaming kernel; every wait (copies and
// MMAs) is bounded and gives up with HY_FAULT_STREAM_* / HY_FAULT_TC_CONV in
// the device fault word.  Two CTAs per SM: one CTA's MMAs run while the
// other does its SIMT work.
#include <cuda_bf16.h>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels.h"
#include "resident.cuh"
#include "status.h"
#include "tcgen05.cuh"
#include "twiddle.h"

namespace hy {

namespace {

constexpr int TC_LOG_M = 13, TC_LOG_P = 5;
constexpr int TC_M = 1 << TC_LOG_M, TC_P = 1 << TC_LOG_P, TC_T = TC_M / TC_P;   // 8192, 32, 256
constexpr int TC_L = TC_M;                                                      // causal: L = M samples
constexpr uint32_t TC_ROW_BYTES = TC_L * 2;                                     // bf16 row
constexpr uint32_t A_PART = TC_T * 128;                                         // 32 KB: 256 rows x 128 B
constexpr uint32_t SBUF_BYTES = ((uint32_t)spad_size(TC_M) * 8 + 1023) & ~1023u;   // exchange buffer, 1 KB aligned
constexpr uint32_t B_PART = 32 * 128;                                           // 4 KB: 32 rows x 128 B
constexpr uint32_t TAB_BYTES = 2 * B_PART;                                      // hi, lo
constexpr size_t TC_SMEM = 1024 + SBUF_BYTES + TAB_BYTES + 2 * (size_t)TC_ROW_BYTES;
constexpr uint32_t TMEM_COLS = 128;                                             // 2 tiles x (32 Re + 32 Im)
constexpr uint32_t IDESC_P = tc::idesc_f16(128, 32, true, false, false);
constexpr uint32_t IDESC_N = tc::idesc_f16(128, 32, true, false, true);         // negated B

static_assert(2 * A_PART <= SBUF_BYTES, "the A operand must fit in the exchange buffer");
static_assert(TC_SMEM <= 113 * 1024, "two CTAs per SM");

// The DFT-32 operand in its shared-memory layout (hi then lo), built on the
// host; copied into each CTA's shared memory once.
__device__ uint4 g_dft32_tab[TAB_BYTES / 16];

// byte offset of 16-byte chunk j of K-major row r (128-byte rows, 128-byte swizzle)
__host__ __device__ constexpr uint32_t sw128(uint32_t r, uint32_t j) {
    return (r >> 3) * 1024u + (r & 7u) * 128u + ((j ^ (r & 7u)) << 4);
}

__device__ __forceinline__ uint32_t bits_bf162(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t *>(&h); }

// x = hi + lo with hi = rn_bf16(x), lo = rn_bf16(x - hi), for a pair (a, b)
__device__ __forceinline__ void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const uint32_t h = bits_bf162(__floats2bfloat162_rn(a, b));
    const float ha = __uint_as_float(h << 16), hb = __uint_as_float(h & 0xffff0000u);
    hi = h;
    lo = bits_bf162(__floats2bfloat162_rn(a - ha, b - hb));
}

// Writes row t of the A operand (hi and lo parts) from the 32 complex values
// y[0..31]: K elements 0..31 = Re y, 32..63 = Im y.
__device__ __forceinline__ void write_a_row(uint8_t *a_base, int t, const float2 (&y)[TC_P]) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {                    // 16-byte chunk j: K elements 8j .. 8j+7
        uint32_t h[4], l[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 8 * j + 2 * e;             // element pair (k, k+1)
            const float a = k < 32 ? y[k].x : y[k - 32].y;
            const float b = k < 32 ? y[k + 1].x : y[k - 31].y;
            split2(a, b, h[e], l[e]);
        }
        const uint32_t off = sw128((uint32_t)t, (uint32_t)j);
        *reinterpret_cast<uint4 *>(a_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(a_base + A_PART + off) = make_uint4(l[0], l[1], l[2], l[3]);
    }
}

// Issues the MMAs of one radix-32 stage (thread 0 only) and commits them to bar.
//   terms: hi·F_hi + hi·F_lo (+ lo·F_hi unless the data is exact)
//   pruned: only the first 16 inputs of each butterfly are non-zero
template <int DIR, bool EXACT, bool PRUNED>
__device__ __forceinline__ void issue_stage_mmas(uint32_t tmem, uint32_t a_addr, uint32_t b_addr, uint64_t *bar) {
    tc::fence_after();
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
        const uint32_t d_re = tmem + 64u * tile, d_im = d_re + 32u;
        const uint64_t a_hi = tc::desc_k_sw128(a_addr + tile * 16384u);
        const uint64_t a_lo = tc::desc_k_sw128(a_addr + A_PART + tile * 16384u);
        const uint64_t b_hi = tc::desc_k_sw128(b_addr), b_lo = tc::desc_k_sw128(b_addr + B_PART);
        constexpr int NTERM = EXACT ? 2 : 3;
        bool first_re = true, first_im = true;
#pragma unroll
        for (int term = 0; term < NTERM; ++term) {
            const uint64_t A = term == 2 ? a_lo : a_hi;
            const uint64_t B = term == 1 ? b_lo : b_hi;
            // K steps of 16 elements (2 descriptor units of 16 bytes each)
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                if (PRUNED && s == 1) continue;
                // Re: Re a · C (steps 0,1 with B steps 0,1) and Im a · S (steps 2,3 with B steps 2,3)
                tc::mma_f16(d_re, A + 2 * s, B + 2 * s, IDESC_P, first_re ? 0u : 1u);
                first_re = false;
                tc::mma_f16(d_re, A + 2 * (s + 2), B + 2 * (s + 2), DIR < 0 ? IDESC_P : IDESC_N, 1u);
                // Im: Im a · C (A steps 2,3 with B steps 0,1) and -+ Re a · S (A steps 0,1 with B steps 2,3)
                tc::mma_f16(d_im, A + 2 * (s + 2), B + 2 * s, IDESC_P, first_im ? 0u : 1u);
                first_im = false;
                tc::mma_f16(d_im, A + 2 * s, B + 2 * (s + 2), DIR < 0 ? IDESC_N : IDESC_P, 1u);
            }
        }
    }
    tc::commit(bar);
}

// All threads: waits for the stage's MMAs, then reads row t's 32 outputs
// (natural order) into y.
__device__ __forceinline__ bool read_stage(uint32_t tmem, int t, uint64_t *bar, uint32_t parity, float2 (&y)[TC_P],
                                           uint32_t *fault) {
    const bool ok = mbar_wait(bar, parity);
    if (!ok) record_fault(fault, HY_FAULT_TC_CONV);
    __syncwarp();                                  // tcgen05.ld is warp-wide (.sync.aligned)
    tc::fence_after();
    const int warp = t >> 5;
    const uint32_t taddr = tmem + ((uint32_t)((warp & 3) * 32) << 16) + 64u * (uint32_t)(warp >> 2);
    uint32_t re[32], im[32];
    tc::tmem_ld32(taddr, re);
    tc::tmem_ld32(taddr + 32u, im);
    tc::tmem_wait_ld();
#pragma unroll
    for (int r = 0; r < TC_P; ++r) y[r] = make_float2(__uint_as_float(re[r]), __uint_as_float(im[r]));
    return ok;
}

// The two output layouts of the radix-32 stages (see fft_stage): stage 0
// writes butterfly t's output r' to element 32 t + r'; stage 1 (p = 32) to
// element (t - k) * 32 + k + 32 r', k = t mod 32.
template <int S>
__device__ __forceinline__ void write_stage_out(float2 *sbuf, int t, const float2 (&y)[TC_P]) {
    if constexpr (S == 0) {
        float2 *dst = sbuf + spad(32 * t);
#pragma unroll
        for (int r = 0; r < TC_P; ++r) dst[r] = y[r];
    } else {
        const int k = t & 31;
        float2 *dst = sbuf + spad((t - k) * 32 + k);
#pragma unroll
        for (int r = 0; r < TC_P; ++r) dst[r * 33] = y[r];
    }
}

template <bool PF_GATE>
__global__ void __launch_bounds__(TC_T, 2) resident_tc_kernel(const ResidentParams p) {
    using IOT = IOTraits<__nv_bfloat16>;
    constexpr int PIN = TC_P / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float2 *sbuf = reinterpret_cast<float2 *>(base);
    uint8_t *a_op = base;                                          // aliases sbuf during the MMAs
    uint8_t *b_tab = base + SBUF_BYTES;
    __nv_bfloat16 *in_st = reinterpret_cast<__nv_bfloat16 *>(b_tab + TAB_BYTES);
    __nv_bfloat16 *g_st = in_st + TC_L;
    __shared__ uint64_t bars[2], mma_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const __nv_bfloat16 *ubase = reinterpret_cast<const __nv_bfloat16 *>(p.u);
    const __nv_bfloat16 *gbase = reinterpret_cast<const __nv_bfloat16 *>(p.gate[0]);
    __nv_bfloat16 *ybase = reinterpret_cast<__nv_bfloat16 *>(p.y);
    const bool gate_pf = PF_GATE && gbase != nullptr;
    auto row_of = [&](int64_t c) { return p.remap ? (c % p.B) * (int64_t)p.D + c / p.B : c; };

    if ((threadIdx.x >> 5) == 0) tc::tmem_alloc(&s_tmem, TMEM_COLS);
    for (int i = threadIdx.x; i < (int)(TAB_BYTES / 16); i += TC_T)
        reinterpret_cast<uint4 *>(b_tab)[i] = g_dft32_tab[i];
    fence_proxy_async_smem();                                      // the table is read by the tensor cores
    int64_t c = blockIdx.x;
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&mma_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t a_addr = smem_u32(a_op), b_addr = smem_u32(b_tab);
    if (threadIdx.x == 0 && c < p.n_rows) bulk_g2s(in_st, ubase + row_of(c) * TC_L, TC_ROW_BYTES, &bars[0]);
    uint32_t w_in = 0, w_g = 0, mph = 0;
    for (; c < p.n_rows; c += gridDim.x) {
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
        // the 16 non-zero inputs of butterfly t: packed pairs (s[2n], s[2n+1]), n = t + 256 m
        uint32_t win[PIN];
#pragma unroll
        for (int m = 0; m < PIN; ++m) win[m] = *reinterpret_cast<const uint32_t *>(in_st + 2 * (t + m * TC_T));
        __syncthreads();                                           // stage buffers free for the next copies
        if (s_abort) break;
        if (t == 0) {
            fence_proxy_async_smem();
            if (gate_pf) bulk_g2s(g_st, gbase + row * TC_L, TC_ROW_BYTES, &bars[1]);
            if (c + gridDim.x < p.n_rows) bulk_g2s(in_st, ubase + row_of(c + gridDim.x) * TC_L, TC_ROW_BYTES, &bars[0]);
        }

        float2 x[TC_P];
        // ---- forward stage 0 on the tensor cores: exact bf16 inputs, K = 16 + 16
        {
#pragma unroll
            for (int j = 0; j < 2; ++j) {                          // Re (chunks 0,1) and Im (chunks 4,5), r = 8j .. 8j+7
                uint32_t re[4], im[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    re[e] = __byte_perm(win[8 * j + 2 * e], win[8 * j + 2 * e + 1], 0x5410);
                    im[e] = __byte_perm(win[8 * j + 2 * e], win[8 * j + 2 * e + 1], 0x7632);
                }
                *reinterpret_cast<uint4 *>(a_op + sw128((uint32_t)t, (uint32_t)j)) = make_uint4(re[0], re[1], re[2], re[3]);
                *reinterpret_cast<uint4 *>(a_op + sw128((uint32_t)t, (uint32_t)(j + 4))) =
                    make_uint4(im[0], im[1], im[2], im[3]);
            }
            fence_proxy_async_smem();
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<-1, true, true>(tmem, a_addr, b_addr, &mma_bar);
            if (!read_stage(tmem, t, &mma_bar, mph, x, p.fault)) s_abort = 1;
            mph ^= 1;
            write_stage_out<0>(sbuf, t, x);
            tc::fence_before();
            __syncthreads();
            load_own<TC_LOG_M, TC_LOG_P>(x, sbuf, t);
            __syncthreads();
        }
        // ---- stages 1 (tensor cores, twiddled) and 2 (SIMT radix 8), forward
        auto tc_stage1 = [&](auto dirc) {
            constexpr int DIR = decltype(dirc)::value;
            const float2 *tw1 = p.tw_fft + plan_tw_offset(TC_LOG_M, TC_LOG_P, 1);
            const int k = t & 31;
#pragma unroll
            for (int r = 1; r < TC_P; ++r) x[r] = cmul_dir<DIR>(x[r], __ldg(tw1 + (r - 1) * 32 + k));
            write_a_row(a_op, t, x);
            fence_proxy_async_smem();
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<DIR, false, false>(tmem, a_addr, b_addr, &mma_bar);
            if (!read_stage(tmem, t, &mma_bar, mph, x, p.fault)) s_abort = 1;
            mph ^= 1;
            write_stage_out<1>(sbuf, t, x);
            tc::fence_before();
            __syncthreads();
            load_own<TC_LOG_M, TC_LOG_P>(x, sbuf, t);
            __syncthreads();
        };
        tc_stage1(std::integral_constant<int, -1>{});
        fft_stage<TC_LOG_M, TC_LOG_P, 2, -1, false>(x, sbuf, t, p.tw_fft + plan_tw_offset(TC_LOG_M, TC_LOG_P, 2),
                                                     SyncBlock{});

        // ---- spectrum product (skip term folded in), real-FFT split / merge
        const float dk = p.skip[0] ? ldv(p.skip[0] + ch) : 0.f;
        const float2 *H = p.spec[0] + smp * p.spec_batch_stride + ch * p.spec_row_stride;
        split_multiply_merge<TC_LOG_M, TC_LOG_P>(x, sbuf, t, H, p.tw_split, dk);

        // ---- inverse: stage 0 (tensor cores, no twiddle), 1 (tensor cores), 2 (SIMT)
        {
            write_a_row(a_op, t, x);
            fence_proxy_async_smem();
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<+1, false, false>(tmem, a_addr, b_addr, &mma_bar);
            if (!read_stage(tmem, t, &mma_bar, mph, x, p.fault)) s_abort = 1;
            mph ^= 1;
            write_stage_out<0>(sbuf, t, x);
            tc::fence_before();
            __syncthreads();
            load_own<TC_LOG_M, TC_LOG_P>(x, sbuf, t);
            __syncthreads();
        }
        tc_stage1(std::integral_constant<int, +1>{});
        fft_stage<TC_LOG_M, TC_LOG_P, 2, +1, false>(x, sbuf, t, p.tw_fft + plan_tw_offset(TC_LOG_M, TC_LOG_P, 2),
                                                     SyncBlock{});

        if (gate_pf) {
            if (!mbar_wait(&bars[1], w_g & 1)) {
                record_fault(p.fault, HY_FAULT_STREAM_GATE);
                s_abort = 1;
            }
            ++w_g;
        }
        __nv_bfloat16 *yout = ybase + row * (int64_t)TC_L;
#pragma unroll
        for (int m = 0; m < PIN; ++m) {
            const int i0 = 2 * (t + m * TC_T);
            float2 z = make_float2(x[m].x * p.scale, x[m].y * p.scale);
            if (gbase) {
                float2 gv;
                if (gate_pf) {
                    const uint32_t b = *reinterpret_cast<const uint32_t *>(g_st + i0);
                    gv = make_float2(__uint_as_float(b << 16), __uint_as_float(b & 0xffff0000u));
                } else {
                    gv = IOT::load2(gbase + row * (int64_t)TC_L + i0);
                }
                z = make_float2(z.x * gv.x, z.y * gv.y);
            }
            IOT::store2(yout + i0, z);
        }
    }
    // no copy may still be landing and no MMA still running when the CTA exits
    if (threadIdx.x == 0) {
        if (w_in && !mbar_wait(&bars[0], (w_in - 1) & 1)) record_fault(p.fault, HY_FAULT_STREAM_INPUT);
        if (w_g && !mbar_wait(&bars[1], (w_g - 1) & 1)) record_fault(p.fault, HY_FAULT_STREAM_GATE);
        tc::commit(&mma_bar);
        if (!mbar_wait(&mma_bar, mph)) record_fault(p.fault, HY_FAULT_TC_CONV);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    __syncwarp();
    if ((threadIdx.x >> 5) == 0) tc::tmem_free(tmem, TMEM_COLS);
}

// ---------------------------------------------------------------- host side
std::mutex g_mu;
bool g_tab_ready[64] = {};
bool g_attr_ready[64] = {};

uint16_t bf16_rn(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}
float bf16_to_float(uint16_t h) {
    const uint32_t u = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

// The operand rows r' = 0..31: [cos(2π r r'/32) r < 32 | sin(2π r r'/32) r < 32],
// split into bf16 hi and lo, in the 128-byte-swizzled K-major layout.
hy_status upload_table(int dev) {
    std::vector<uint16_t> tab(TAB_BYTES / 2, 0);
    for (int rp = 0; rp < 32; ++rp)
        for (int k = 0; k < 64; ++k) {
            const int r = k & 31;
            const int e = (r * rp) & 31;                      // exact angle reduction
            const double ang = 2.0 * 3.14159265358979323846264338327950288 * e / 32.0;
            const double v = k < 32 ? std::cos(ang) : std::sin(ang);
            const uint16_t hi = bf16_rn((float)v);
            const uint16_t lo = bf16_rn((float)(v - (double)bf16_to_float(hi)));
            const uint32_t off = sw128((uint32_t)rp, (uint32_t)(k >> 3)) + 2u * (uint32_t)(k & 7);
            tab[off / 2] = hi;
            tab[(B_PART + off) / 2] = lo;
        }
    void *dst = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&dst, g_dft32_tab);
    if (e != cudaSuccess) return set_cuda_error("tensor-core DFT table address", e);
    e = cudaMemcpy(dst, tab.data(), TAB_BYTES, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return set_cuda_error("tensor-core DFT table upload", e);
    g_tab_ready[dev] = true;
    return HY_OK;
}

}  // namespace

bool resident_tc_eligible(const ResidentParams &p, int log_m, hy_dtype dt, bool circular) {
    return dt == HY_BF16 && !circular && p.K == 1 && log_m == TC_LOG_M && p.L == TC_L &&
           ((uintptr_t)p.u & 15u) == 0 && ((uintptr_t)p.y & 15u) == 0 &&
           (!p.gate[0] || ((uintptr_t)p.gate[0] & 15u) == 0);
}

hy_status launch_resident_tc(ResidentParams p, cudaStream_t s) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return set_error(HY_ERR_UNSUPPORTED, "device index %d >= 64", dev);
    constexpr bool PF = true;
    auto kernel = resident_tc_kernel<PF>;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_tab_ready[dev]) {
            hy_status st = upload_table(dev);
            if (st != HY_OK) return st;
        }
        if (!g_attr_ready[dev]) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TC_SMEM);
            if (e != cudaSuccess) return set_cuda_error("tensor-core conv smem attribute", e);
            g_attr_ready[dev] = true;
        }
    }
    p.tw_fft = tw_stages(TC_LOG_M, TC_LOG_P);
    p.tw_split = tw_split(TC_LOG_M);
    if (!p.tw_fft || !p.tw_split) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^13");
    p.fault = device_fault_word();
    if (!p.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, TC_T, TC_SMEM);
    if (e != cudaSuccess) return set_cuda_error("occupancy query", e);
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)per_sm * device_sm_count();
    if (grid > p.n_rows) grid = p.n_rows;
    kernel<<<(unsigned)grid, TC_T, TC_SMEM, s>>>(p);
    return check_launch("tensor-core conv launch");
}

}  // namespace hy
