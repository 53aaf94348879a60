// resident_tc.cu -- the streaming FFT convolution of one order with the two
// radix-32 stages of each FFT done as DFT matrix products on the tcgen05
// tensor cores: rows of L = 8192 bf16 samples (M = 8192 complex points, the
// order-2 operator at its ~153M-model width and 8K length), causal.
//
// The transform plan is the on-chip kernel's (resident.cuh): Stockham stages
// of radix 32, 32 and 8 over M = 8192, 256 threads, thread t owning elements
// t + 256 m.  In a radix-32 stage every thread holds the 32 inputs of one
// butterfly, so the 256 butterflies of a stage are one matrix product
//   D[t, r'] = Σ_r a_t[r] · W_32^{r r'}
// on 2 M-tiles of 128 rows.  Complex values are carried as real K-blocks:
// the A row of butterfly t is [Re a_t[0..31] | Im a_t[0..31]] (K = 64) and
// the constant operand has one row per real output: rows r' < 32 give
// Re D = Re a·C + Im a·S and rows 32 + r' give Im D = −Re a·S + Im a·C
// (C = cos(2π r r'/32), S = sin(2π r r'/32)), so one M = 128, N = 64, K = 16
// MMA per K step computes both parts.  The inverse transform uses the same
// operand through conj(DFT(conj a)): the imaginary parts of the A rows and
// of the results are negated.
//
// The A operand lives in tensor memory: thread t writes its own row with
// tcgen05.st (lane t % 128 of tile t / 128, two bf16 per 32-bit column), and
// the MMAs read it from there, so the butterfly operands cost no shared-memory
// bandwidth.  The accumulators are TMEM columns too (Re at 0..31, Im at
// 32..63 of each tile); thread t reads its row back with tcgen05.ld.  TMEM
// per CTA: 128 accumulator + 128 operand columns (hi and lo parts).
//
// Precision: every fp32 operand x is split into bf16 parts hi = rn(x),
// lo = rn(x − hi), and products are summed as hi·hi + hi·lo + lo·hi with
// fp32 accumulation (relative error of each product about 2^-17; the
// dropped lo·lo term is smaller).  The first forward stage takes the bf16
// input samples themselves, which are exact, so it needs only hi·(F_hi +
// F_lo), and only the 16 non-zero inputs of each butterfly (the zero-padded
// half) are multiplied.  The radix-8 stage, the twiddles, the real-FFT split
// / merge with the spectrum product (and skip term), the gate and the bf16
// rounding of the output are the fp32 SIMT code of resident.cuh.
//
// Rows are staged by TMA bulk copies on mbarriers as in the streaming
// kernel; the gate is read in the epilogue.  Every wait (copies and MMAs) is
// bounded and gives up with HY_FAULT_STREAM_INPUT / HY_FAULT_TC_CONV in the
// device fault word.  Two CTAs per SM: one CTA's MMAs run while the other
// does its SIMT work.
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
constexpr uint32_t B_PART = 64 * 128;                                           // 8 KB: 64 rows x 128 B
constexpr uint32_t TAB_BYTES = 2 * B_PART;                                      // hi, lo
constexpr uint32_t SBUF_BYTES = ((uint32_t)spad_size(TC_M) * 8 + 15) & ~15u;    // exchange buffer
constexpr size_t TC_SMEM = 1024 + TAB_BYTES + SBUF_BYTES + (size_t)TC_ROW_BYTES;
constexpr uint32_t TMEM_COLS = 256;     // [0,128): accumulators, [128,192): A hi, [192,256): A lo (2 tiles each)
constexpr uint32_t COL_A_HI = 128, COL_A_LO = 192;
constexpr uint32_t IDESC = tc::idesc_f16(128, 64, true);

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

// TMEM address of this thread's row (lane t % 128 of tile t / 128) at column col
__device__ __forceinline__ uint32_t row_addr(uint32_t tmem, int t, uint32_t col_of_tile0, uint32_t tile_stride) {
    const int warp = t >> 5;
    return tmem + ((uint32_t)((warp & 3) * 32) << 16) + col_of_tile0 + tile_stride * (uint32_t)(warp >> 2);
}

// Writes row t of the A operand (hi and lo parts) into TMEM from the 32
// complex values y[0..31] (conjugated when CONJ): K elements 0..31 = Re y,
// 32..63 = Im y, two per 32-bit column.
template <bool CONJ>
__device__ __forceinline__ void write_a_row(uint32_t tmem, int t, const float2 (&y)[TC_P]) {
    uint32_t h[32], l[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        split2(y[2 * j].x, y[2 * j + 1].x, h[j], l[j]);
        if (CONJ) split2(-y[2 * j].y, -y[2 * j + 1].y, h[16 + j], l[16 + j]);
        else split2(y[2 * j].y, y[2 * j + 1].y, h[16 + j], l[16 + j]);
    }
    tc::tmem_st32(row_addr(tmem, t, COL_A_HI, 32), h);
    tc::tmem_st32(row_addr(tmem, t, COL_A_LO, 32), l);
    tc::tmem_wait_st();
}

// Issues the MMAs of one radix-32 stage (thread 0 only) and commits them to bar.
//   terms: hi·F_hi + hi·F_lo (+ lo·F_hi unless the data is exact)
//   pruned: only the first 16 inputs of each butterfly are non-zero (K steps 0 and 2)
template <bool EXACT, bool PRUNED>
__device__ __forceinline__ void issue_stage_mmas(uint32_t tmem, uint32_t b_addr, uint64_t *bar) {
    tc::fence_after();
    const uint64_t b_hi = tc::desc_k_sw128(b_addr), b_lo = tc::desc_k_sw128(b_addr + B_PART);
    constexpr int NTERM = EXACT ? 2 : 3;
#pragma unroll
    for (int tile = 0; tile < 2; ++tile) {
        const uint32_t d = tmem + 64u * tile;
        bool first = true;
#pragma unroll
        for (int term = 0; term < NTERM; ++term) {
            const uint32_t a = tmem + (term == 2 ? COL_A_LO : COL_A_HI) + 32u * tile;
            const uint64_t B = term == 1 ? b_lo : b_hi;
#pragma unroll
            for (int s = 0; s < 4; ++s) {                // K step of 16 elements: 8 TMEM columns, 32 B of B
                if (PRUNED && (s & 1)) continue;
                tc::mma_f16_ts(d, a + 8u * s, B + 2 * s, IDESC, first ? 0u : 1u);
                first = false;
            }
        }
    }
    tc::commit(bar);
}

// Thread 0 waits for the stage's MMAs (the others are parked at the CTA
// barrier instead of polling, so they issue nothing meanwhile and the other
// CTA on the SM gets the issue slots); then every thread reads row t's 32
// outputs (natural order; conjugated when CONJ) into y.
template <bool CONJ>
__device__ __forceinline__ void read_stage(uint32_t tmem, int t, uint64_t *bar, uint32_t parity, float2 (&y)[TC_P],
                                           uint32_t *fault, int *abort_flag) {
    if (t == 0 && !mbar_wait_sleep(bar, parity)) {
        record_fault(fault, HY_FAULT_TC_CONV);
        *abort_flag = 1;
    }
    __syncthreads();
    tc::fence_after();
    const uint32_t taddr = row_addr(tmem, t, 0, 64);
    uint32_t re[32], im[32];
    tc::tmem_ld32(taddr, re);
    tc::tmem_ld32(taddr + 32u, im);
    tc::tmem_wait_ld();
#pragma unroll
    for (int r = 0; r < TC_P; ++r)
        y[r] = make_float2(__uint_as_float(re[r]), CONJ ? -__uint_as_float(im[r]) : __uint_as_float(im[r]));
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

__global__ void __launch_bounds__(TC_T, 2) resident_tc_kernel(const ResidentParams p) {
    using IOT = IOTraits<__nv_bfloat16>;
    constexpr int PIN = TC_P / 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *b_tab = base;                                          // 1024-byte aligned swizzle atoms
    float2 *sbuf = reinterpret_cast<float2 *>(base + TAB_BYTES);
    __nv_bfloat16 *in_st = reinterpret_cast<__nv_bfloat16 *>(base + TAB_BYTES + SBUF_BYTES);
    __shared__ uint64_t in_bar, mma_bar;
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort;

    const __nv_bfloat16 *ubase = reinterpret_cast<const __nv_bfloat16 *>(p.u);
    const __nv_bfloat16 *gbase = reinterpret_cast<const __nv_bfloat16 *>(p.gate[0]);
    __nv_bfloat16 *ybase = reinterpret_cast<__nv_bfloat16 *>(p.y);
    auto row_of = [&](int64_t c) { return p.remap ? (c % p.B) * (int64_t)p.D + c / p.B : c; };

    if ((threadIdx.x >> 5) == 0) tc::tmem_alloc(&s_tmem, TMEM_COLS);
    for (int i = threadIdx.x; i < (int)(TAB_BYTES / 16); i += TC_T)
        reinterpret_cast<uint4 *>(b_tab)[i] = g_dft32_tab[i];
    fence_proxy_async_smem();                                      // the table is read by the tensor cores
    int64_t c = blockIdx.x;
    if (threadIdx.x == 0) {
        mbar_init(&in_bar, 1);
        mbar_init(&mma_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s_tmem;
    const uint32_t b_addr = smem_u32(b_tab);
    if (threadIdx.x == 0 && c < p.n_rows) bulk_g2s(in_st, ubase + row_of(c) * TC_L, TC_ROW_BYTES, &in_bar);
    uint32_t w_in = 0, mph = 0;
    for (; c < p.n_rows; c += gridDim.x) {
        int t;
        asm volatile("mov.u32 %0, %%tid.x;" : "=r"(t));
        const int64_t row = row_of(c);
        const int64_t ch = (row / p.sdiv) % p.smod;
        const int64_t smp = row / (p.sdiv * p.smod);
        if (!mbar_wait(&in_bar, w_in & 1)) {
            record_fault(p.fault, HY_FAULT_STREAM_INPUT);
            s_abort = 1;
        }
        ++w_in;
        // the 16 non-zero inputs of butterfly t: packed pairs (s[2n], s[2n+1]), n = t + 256 m
        uint32_t win[PIN];
#pragma unroll
        for (int m = 0; m < PIN; ++m) win[m] = *reinterpret_cast<const uint32_t *>(in_st + 2 * (t + m * TC_T));
        __syncthreads();                                           // the stage buffer is free for the next copy
        if (s_abort) break;
        if (t == 0 && c + gridDim.x < p.n_rows) {
            fence_proxy_async_smem();
            bulk_g2s(in_st, ubase + row_of(c + gridDim.x) * TC_L, TC_ROW_BYTES, &in_bar);
        }

        float2 x[TC_P];
        // ---- forward stage 0 on the tensor cores: exact bf16 inputs, K steps 0 (Re) and 2 (Im)
        {
            uint32_t re[8], im[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                re[e] = __byte_perm(win[2 * e], win[2 * e + 1], 0x5410);
                im[e] = __byte_perm(win[2 * e], win[2 * e + 1], 0x7632);
            }
            tc::tmem_st8(row_addr(tmem, t, COL_A_HI, 32), re);
            tc::tmem_st8(row_addr(tmem, t, COL_A_HI + 16, 32), im);
            tc::tmem_wait_st();
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<true, true>(tmem, b_addr, &mma_bar);
            read_stage<false>(tmem, t, &mma_bar, mph, x, p.fault, &s_abort);
            mph ^= 1;
            write_stage_out<0>(sbuf, t, x);
            tc::fence_before();
            __syncthreads();
            load_own<TC_LOG_M, TC_LOG_P>(x, sbuf, t);
            __syncthreads();
        }
        // ---- stage 1 (tensor cores, twiddled); the inverse works on conjugates
        auto tc_stage1 = [&](auto dirc) {
            constexpr int DIR = decltype(dirc)::value;
            const float2 *tw1 = p.tw_fft + plan_tw_offset(TC_LOG_M, TC_LOG_P, 1);
            const int k = t & 31;
            // forward: a = x w; inverse: conj(x conj(w)) = conj(x) w, written as is
#pragma unroll
            for (int r = 1; r < TC_P; ++r) {
                const float2 w = __ldg(tw1 + (r - 1) * 32 + k);
                x[r] = DIR < 0 ? cmul(x[r], w) : cmul(cconj(x[r]), w);
            }
            if (DIR > 0) x[0] = cconj(x[0]);
            write_a_row<false>(tmem, t, x);
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<false, false>(tmem, b_addr, &mma_bar);
            read_stage<(DIR > 0)>(tmem, t, &mma_bar, mph, x, p.fault, &s_abort);
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
            write_a_row<true>(tmem, t, x);
            tc::fence_before();
            __syncthreads();
            if (t == 0) issue_stage_mmas<false, false>(tmem, b_addr, &mma_bar);
            read_stage<true>(tmem, t, &mma_bar, mph, x, p.fault, &s_abort);
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

        // ---- epilogue: scale, gate (read here), bf16 store of the first L samples
        __nv_bfloat16 *yout = ybase + row * (int64_t)TC_L;
        const __nv_bfloat16 *grow = gbase ? gbase + row * (int64_t)TC_L : nullptr;
        constexpr int EB = 8;
#pragma unroll
        for (int m0 = 0; m0 < PIN; m0 += EB) {
            float2 gv[EB];
#pragma unroll
            for (int j = 0; j < EB; ++j)
                gv[j] = grow ? IOT::load2(grow + 2 * (t + (m0 + j) * TC_T)) : make_float2(1.f, 1.f);
#pragma unroll
            for (int j = 0; j < EB; ++j) {
                const int m = m0 + j;
                const int i0 = 2 * (t + m * TC_T);
                IOT::store2(yout + i0, make_float2(x[m].x * p.scale * gv[j].x, x[m].y * p.scale * gv[j].y));
            }
        }
    }
    // no copy may still be landing and no MMA still running when the CTA exits
    if (threadIdx.x == 0) {
        if (w_in && !mbar_wait(&in_bar, (w_in - 1) & 1)) record_fault(p.fault, HY_FAULT_STREAM_INPUT);
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

// The operand rows: n < 32 give Re of output n, [cos(2π r n/32) | sin(2π r n/32)]
// over r = 0..31; n = 32 + n' give Im of output n', [-sin | cos]; split into
// bf16 hi and lo, in the 128-byte-swizzled K-major layout.
hy_status upload_table(int dev) {
    std::vector<uint16_t> tab(TAB_BYTES / 2, 0);
    for (int n = 0; n < 64; ++n)
        for (int k = 0; k < 64; ++k) {
            const int r = k & 31, o = n & 31;
            const int e = (r * o) & 31;                       // exact angle reduction
            const double ang = 2.0 * 3.14159265358979323846264338327950288 * e / 32.0;
            const double c = std::cos(ang), sn = std::sin(ang);
            const double v = n < 32 ? (k < 32 ? c : sn) : (k < 32 ? -sn : c);
            const uint16_t hi = bf16_rn((float)v);
            const uint16_t lo = bf16_rn((float)(v - (double)bf16_to_float(hi)));
            const uint32_t off = sw128((uint32_t)n, (uint32_t)(k >> 3)) + 2u * (uint32_t)(k & 7);
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
    auto kernel = resident_tc_kernel;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_tab_ready[dev]) {
            hy_status st = upload_table(dev);
            if (st != HY_OK) return st;
        }
        if (!g_attr_ready[dev]) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TC_SMEM);
            if (e != cudaSuccess) return set_cuda_error("tensor-core conv smem attribute", e);
            // the largest shared-memory carve-out: two CTAs per SM fit only in it
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return set_cuda_error("tensor-core conv carve-out attribute", e);
            g_attr_ready[dev] = true;
        }
    }
    p.tw_fft = tw_stages(TC_LOG_M, TC_LOG_P);
    p.tw_split = tw_split(TC_LOG_M);
    if (!p.tw_fft || !p.tw_split) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^13");
    p.fault = device_fault_word();
    if (!p.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
    // Two CTAs per SM: registers (128 x 256 threads), shared memory (<= 113 KB
    // with the largest carve-out) and TMEM (256 columns) are sized for that.
    // (The occupancy query answers 1 for this kernel; with a grid of 2 per SM
    // the rows are spread over both resident CTAs.)
    const int64_t grid = 2 * (int64_t)device_sm_count() < p.n_rows ? 2 * (int64_t)device_sm_count() : p.n_rows;
    kernel<<<(unsigned)grid, TC_T, TC_SMEM, s>>>(p);
    return check_launch("tensor-core conv launch");
}

}  // namespace hy
