// fourstep.cu -- multi-pass FFT convolution for sequences too long for one
// CTA ([HN] step 3 chain and [ES] FFT convolution at HyenaDNA-scale length).
//
// A row of n = 2M real samples is packed into M = N1*N2 complex points
// z[m] = s[2m] + i s[2m+1] (zero for m >= M/2: the causal zero-padding).  With
// input index m = n1 + N1*n2 and bin index k = k2 + N2*k1:
//
//   Z[k2 + N2 k1] = Σ_n1 W_N1^{n1 k1} · W_M^{n1 k2} · Σ_n2 z[n1 + N1 n2] W_N2^{n2 k2}
//
//   pass A (columns): for each n1, FFT over n2, times W_M^{n1 k2}, stored at
//                     n1 + N1*k2 (the input layout).
//   pass B (rows):    for each k2 the N1 values are contiguous: FFT over n1
//                     gives Z at bins k2 + N2*k1.  Bin k pairs with M - k,
//                     which lives in row N2 - k2 (row 0 and row N2/2 pair with
//                     themselves), so a CTA holds 4 rows and their 4 mirrors
//                     and does the real-FFT split, the spectrum product and
//                     the merge there, then the inverse row FFT and
//                     W_M^{-n1 k2}.
//   pass C (columns): inverse FFT over k2, first half of the outputs only,
//                     then the gate; when another order follows, its pass A
//                     runs in the same kernel on the same columns.
//
// The skip term D_k z_k is taken into the product: D_k z_k is the causal
// convolution of z_k with D_k times a unit impulse, whose length-2M DFT is
// D_k at every bin, so pass B multiplies by H_k + D_k instead of H_k and
// nothing else of z_k has to be kept (the rounding of the skip term then
// follows the FFT round trip, a few fp32 ulps of |D_k z_k|).
//
// Each column or row FFT (N1, N2 <= 1024) is done by one warp (block_fft with
// warp synchronisation).  A column pass moves its 8 columns x N2 rows of the
// complex intermediate between global and shared memory as 2-D TMA tensor
// tiles (rows of 64 bytes, 64-byte swizzle, loads completing on an mbarrier
// with a bounded wait, stores as bulk tensor stores), so no thread spends
// registers or instructions on the strided transfer and three CTAs fit on an
// SM.  Rows are processed in chunks whose intermediates (8 bytes per complex
// point) stay resident in the 126 MB L2 between passes.
#include <cstring>
#include <mutex>

#include "../../include/hyena.h"
#include "chunk_lanes.h"
#include "kernels.h"
#include "fft_core.cuh"
#include "status.h"
#include "tcgen05.cuh"
#include "twiddle.h"

namespace hy {

namespace {

constexpr int WARPS = 8;          // columns or rows per CTA
constexpr int NT = WARPS * 32;

__host__ __device__ constexpr int fs_log_p(int log_n) { return log_n - 5; }   // per-lane points

// W_N^e from a two-level table: tab[0..2^lo) = W_N^j, tab[2^lo + j] = W_N^{j 2^lo}
__device__ __forceinline__ float2 tw2(const float2 *__restrict__ tab, int lo, uint32_t e) {
    const float2 a = __ldg(tab + (e & ((1u << lo) - 1)));
    const float2 b = __ldg(tab + (1u << lo) + (e >> lo));
    return cmul(a, b);
}
// The twiddles of a warp's 32 P points e = u (lane + 32 m) (u the same for
// the whole warp) split as W^{u lane} W^{32 u m}: one gather per lane, and per
// m a lookup whose address is the same in every lane (one sector instead of
// up to 32 scattered ones).  Four table entries and three roundings per
// twiddle instead of two and one.

struct FsParams {
    int64_t row0;                 // first row of this chunk (flat b*D + d)
    int64_t D;
    int L;                        // valid real samples per row
    int K, k;                     // orders, current order
    const void *u;                // z_0 rows (IO)
    const void *gate_k;           // x_k of the current order (pass C), IO
    const float *skip_k;          // D_k (pass B: added to every bin of H_k)
    const float2 *spec;           // H of the current order (pass B)
    float2 *buf;                  // ws: complex buffer, chunk_rows x M
    void *y;                      // output (IO)
    float scale;                  // 1 / (2n)
    const float2 *tw_n1;          // block FFT tables (size N1, per-lane 2^(log N1 - 5))
    const float2 *tw_n2;
    const float2 *tw_m;           // two-level W_M
    int lo_m;
    const float2 *tw_2m;          // two-level W_{2M}
    int lo_2m;
    float2 *Hout;                 // spectrum mode: output bins (rows x (M+1))
    int vec4;                     // rows of u, gates and y take 4-element vector accesses
    int in_tma;                   // pass A reads its input tile through imap (fp32 rows of M samples)
    int gate_pf;                  // pass C: imap is the gate's map; its tile is prefetched into L2
    uint32_t *fault;              // device fault word (a tile copy that did not land)
};

// Column tiles in shared memory.  The TMA tile of a column pass is N2 rows x
// 64 bytes (8 complex columns) with the 64-byte swizzle: the 16-byte chunk j
// of row r sits at chunk j ^ ((r >> 1) & 3).  It shares its space with the
// warps' padded FFT exchange buffers (WARPS x spad_size(N2) complex), which
// are larger; the space starts on a 1024-byte boundary.
template <int LOG_N2>
__host__ __device__ constexpr size_t colpass_smem_bytes() {
    return 1024 + sizeof(float2) * (size_t)WARPS * spad_size(1 << LOG_N2);
}
constexpr int kTileBoxRows = 256;    // rows per TMA box (the box limit)
__device__ __forceinline__ int tile_swz(int r, int c) { return 64 * r + ((((c >> 1) ^ (r >> 1)) & 3) << 4) + ((c & 1) << 3); }

// ----------------------------------------------------------------------------
// Column pass: A (forward), C (inverse + epilogue), or C followed by A.
// Block (blockIdx.x = column block of 8, blockIdx.y = row in chunk).
// ----------------------------------------------------------------------------
template <int LOG_N1, int LOG_N2, typename IO, bool INV, bool FWD, bool SPEC_INPUT>
__global__ void __launch_bounds__(NT, 3) colpass_kernel(const FsParams p, const __grid_constant__ CUtensorMap bmap,
                                                        const __grid_constant__ CUtensorMap imap) {
    constexpr int N1 = 1 << LOG_N1;
    constexpr int N2 = 1 << LOG_N2;
    constexpr int M = N1 * N2;
    constexpr int LP = fs_log_p(LOG_N2);
    constexpr int P = 1 << LP;
    constexpr int CS = spad_size(N2);           // column stride in the tile
    using IOT = IOTraits<IO>;

    constexpr int BR = N2 < kTileBoxRows ? N2 : kTileBoxRows;
    extern __shared__ unsigned char smem_raw[];
    __shared__ uint64_t tile_bar;
    unsigned char *tb = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);   // TMA tile
    float2 *tile = reinterpret_cast<float2 *>(tb);   // WARPS padded columns x CS (same space)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n1_0 = blockIdx.x * WARPS;
    const int64_t row = p.row0 + blockIdx.y;
    const int64_t rl = blockIdx.y;              // row within chunk
    const int L = p.L;
    float2 *col = tile + warp * CS;
    float2 x[P];

    // Each thread owns EIT groups of 4 consecutive real samples (2 complex
    // points of neighbouring columns) in the first N2/2 rows.  Global loads
    // are issued for all of a thread's groups before any of them is used.
    constexpr int EIT = (N2 / 2) * (WARPS / 2) / NT;
    static_assert(EIT * NT == (N2 / 2) * (WARPS / 2), "column tile does not divide evenly");
    auto group_of = [&](int i, int &r, int &c2) {
        const int e = tid + i * NT;
        r = e / (WARPS / 2);
        c2 = (e % (WARPS / 2)) * 2;
    };
    // 4 real samples at s0 of a row (zero past L)
    auto load_row4 = [&](auto *src, int64_t s0, bool vec, auto loader1, auto loader4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (vec && s0 + 3 < L) {
            v = loader4(src + s0);
        } else {
            if (s0 + 0 < L) v.x = loader1(src + s0 + 0);
            if (s0 + 1 < L) v.y = loader1(src + s0 + 1);
            if (s0 + 2 < L) v.z = loader1(src + s0 + 2);
            if (s0 + 3 < L) v.w = loader1(src + s0 + 3);
        }
        return v;
    };
    auto io1 = [](const IO *q) { return IOT::load(q); };
    auto io4 = [](const IO *q) { return IOT::load4(q); };
    auto h1 = [](const float *q) { return ldv(q); };
    auto h4 = [](const float *q) { return ldv4(q); };

    if constexpr (INV) {
        // ---- all N2 rows of the 8 columns: one TMA tile (N2 / BR boxes of
        //      16 floats x BR rows at x = 2 n1_0, y = rl N2 + b BR)
        if (tid == 0) {
            mbar_init(&tile_bar, 1);
            mbar_init_fence();
        }
        __syncthreads();
        if (tid == 0) {
            tc::mbar_expect_tx(&tile_bar, (uint32_t)N2 * 64u);
#pragma unroll
            for (int b = 0; b < N2 / BR; ++b)
                tc::tma_load_2d(tb + b * BR * 64, &bmap, 2 * n1_0, (int)(rl * N2 + b * BR), &tile_bar);
            if (p.gate_pf) {
                // the gate tile of the epilogue (the same 8 columns' N2/2 rows) into L2
                constexpr int BRI = (N2 / 2) < kTileBoxRows ? (N2 / 2) : kTileBoxRows;
#pragma unroll
                for (int b = 0; b < (N2 / 2) / BRI; ++b) tc::tma_prefetch_l2_2d(&imap, 2 * n1_0, (int)(row * (N2 / 2) + b * BRI));
            }
        }
        const bool landed = mbar_wait(&tile_bar, 0);
        // column `warp`, rows lane + 32 m: the swizzle term depends on the lane only
        {
            const unsigned char *src = tb + tile_swz(lane, warp);
#pragma unroll
            for (int m = 0; m < P; ++m) x[m] = *reinterpret_cast<const float2 *>(src + 2048 * m);
        }
        if (__syncthreads_or(!landed)) {
            // the tile did not land in time: record it, give the copy one more
            // bounded wait so it does not write into a later CTA's memory, stop
            if (tid == 0) {
                record_fault(p.fault, HY_FAULT_MULTIPASS);
                mbar_wait(&tile_bar, 0);
            }
            return;
        }
        block_fft<LOG_N2, LP, +1, false, SyncWarp>(x, col, lane, p.tw_n2, SyncWarp{});
        // keep the first half (n2 < N2/2): samples 2m, 2m+1 with m < M/2
#pragma unroll
        for (int m = 0; m < P / 2; ++m) col[spad(lane + 32 * m)] = x[m];
        // ---- gate inputs, all requested up front
        const IO *g = reinterpret_cast<const IO *>(p.gate_k);
        const IO *grow = g ? g + row * (int64_t)L : nullptr;
        const bool vec = p.vec4 != 0;
        float4 gv[EIT];
#pragma unroll
        for (int i = 0; i < EIT; ++i) {
            int r, c2;
            group_of(i, r, c2);
            const int64_t s0 = 2 * ((int64_t)n1_0 + c2 + (int64_t)N1 * r);
            gv[i] = grow ? load_row4(grow, s0, vec, io1, io4) : make_float4(1.f, 1.f, 1.f, 1.f);
        }
        __syncthreads();
        // ---- epilogue: 8 columns x N2/2 rows; each thread handles 2 complex
        //      = 4 consecutive real samples at 2*(n1_0 + c2 + N1*r)
        const bool last = (p.k == p.K - 1);
        IO *yout = reinterpret_cast<IO *>(p.y) + row * (int64_t)L;
#pragma unroll
        for (int i = 0; i < EIT; ++i) {
            int r, c2;
            group_of(i, r, c2);
            const int64_t s0 = 2 * ((int64_t)n1_0 + c2 + (int64_t)N1 * r);   // first real sample
            const float2 a = tile[c2 * CS + spad(r)], b = tile[(c2 + 1) * CS + spad(r)];
            const float sc = p.scale;
            float4 v = make_float4(gv[i].x * (a.x * sc), gv[i].y * (a.y * sc), gv[i].z * (b.x * sc),
                                   gv[i].w * (b.y * sc));
            if (s0 + 0 >= L) v.x = 0.f;
            if (s0 + 1 >= L) v.y = 0.f;
            if (s0 + 2 >= L) v.z = 0.f;
            if (s0 + 3 >= L) v.w = 0.f;
            const bool full = s0 + 3 < L;
            if (last) {
                if (vec && full) {
                    IOT::store4(yout + s0, v);
                } else {
                    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (s0 + q < L) IOT::store(yout + s0 + q, vv[q]);
                }
            } else {
                tile[c2 * CS + spad(r)] = make_float2(v.x, v.y);
                tile[(c2 + 1) * CS + spad(r)] = make_float2(v.z, v.w);
            }
        }
        if (last || !FWD) return;
        __syncthreads();
    } else if (p.in_tma) {
        // ---- first order, fp32 rows of exactly M samples: the 8 columns'
        //      N2/2 nonzero rows as one TMA tile of the input viewed as rows
        //      of 2 N1 floats (y = row N2/2 + b BR), read straight into x
        constexpr int BRI = (N2 / 2) < kTileBoxRows ? (N2 / 2) : kTileBoxRows;
        if (tid == 0) {
            mbar_init(&tile_bar, 1);
            mbar_init_fence();
        }
        __syncthreads();
        if (tid == 0) {
            tc::mbar_expect_tx(&tile_bar, (uint32_t)(N2 / 2) * 64u);
#pragma unroll
            for (int b = 0; b < (N2 / 2) / BRI; ++b)
                tc::tma_load_2d(tb + b * BRI * 64, &imap, 2 * n1_0, (int)(row * (N2 / 2) + b * BRI), &tile_bar);
        }
        const bool landed = mbar_wait(&tile_bar, 0);
        {
            const unsigned char *src = tb + tile_swz(lane, warp);
#pragma unroll
            for (int m = 0; m < P; ++m)
                x[m] = m < P / 2 ? *reinterpret_cast<const float2 *>(src + 2048 * m) : make_float2(0.f, 0.f);
        }
        if (__syncthreads_or(!landed)) {
            if (tid == 0) {
                record_fault(p.fault, HY_FAULT_MULTIPASS);
                mbar_wait(&tile_bar, 0);
            }
            return;
        }
    } else {
        // ---- first order: packed input rows n2 < N2/2 of the 8 columns
        float4 v[EIT];
        if constexpr (SPEC_INPUT) {
            const float *hin = reinterpret_cast<const float *>(p.u) + row * (int64_t)L;
#pragma unroll
            for (int i = 0; i < EIT; ++i) {
                int r, c2;
                group_of(i, r, c2);
                v[i] = load_row4(hin, 2 * ((int64_t)n1_0 + c2 + (int64_t)N1 * r), p.vec4 != 0, h1, h4);
            }
        } else {
            const IO *uin = reinterpret_cast<const IO *>(p.u) + row * (int64_t)L;
#pragma unroll
            for (int i = 0; i < EIT; ++i) {
                int r, c2;
                group_of(i, r, c2);
                v[i] = load_row4(uin, 2 * ((int64_t)n1_0 + c2 + (int64_t)N1 * r), p.vec4 != 0, io1, io4);
            }
        }
#pragma unroll
        for (int i = 0; i < EIT; ++i) {
            int r, c2;
            group_of(i, r, c2);
            tile[c2 * CS + spad(r)] = make_float2(v[i].x, v[i].y);
            tile[(c2 + 1) * CS + spad(r)] = make_float2(v[i].z, v[i].w);
        }
        __syncthreads();
    }
    if constexpr (FWD) {
        // ---- forward column FFT (upper half zero) and W_M^{n1 k2}
        if (INV || !p.in_tma) {
            load_own<LOG_N2, LP>(x, col, lane);
            __syncwarp();
        }
        block_fft<LOG_N2, LP, -1, true, SyncWarp>(x, col, lane, p.tw_n2, SyncWarp{});
        // W_M^{n1 k2}, k2 = lane + 32 m
        const uint32_t n1 = n1_0 + warp;
        const float2 tl = tw2(p.tw_m, p.lo_m, (n1 * (uint32_t)lane) & (M - 1));
#pragma unroll
        for (int m = 0; m < P; ++m) x[m] = cmul(x[m], cmul(tl, tw2(p.tw_m, p.lo_m, (32u * n1 * (uint32_t)m) & (M - 1))));
        // ---- back to the buffer as one TMA tile: every warp is done with its
        //      exchange buffer before the tile overwrites them
        __syncthreads();
        {
            unsigned char *dst = tb + tile_swz(lane, warp);
#pragma unroll
            for (int m = 0; m < P; ++m) *reinterpret_cast<float2 *>(dst + 2048 * m) = x[m];
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int b = 0; b < N2 / BR; ++b) tc::tma_store_2d(&bmap, tb + b * BR * 64, 2 * n1_0, (int)(rl * N2 + b * BR));
            tc::bulk_commit();
            tc::bulk_wait_all();
        }
    }
}

// ----------------------------------------------------------------------------
// Row pass (B): 8 rows per CTA -- 4 low rows k2 and their mirrors N2 - k2
// (group 0: rows 0..3, N2/2, N2-1..N2-3).  SPEC: write the half spectrum of
// the rows instead of multiplying (long filter spectra).
//
// Bin k = k2 + N2 k1 of a low row pairs with bin M - k = (N2 - k2) + N2 (N1 -
// 1 - k1) of its mirror row, so every warp takes the pairs of its own bins
// k1 < N1/2 (partner values read from the mirror row in shared memory); rows
// 0 and N2/2 pair with themselves.
//
// One row alone touches one 8-byte value per 32-byte sector of a natural-
// order spectrum.  The CTA's rows come in runs of 4 consecutive k2, so the
// spectrum bins are staged in shared memory by all 256 threads with 4
// neighbouring lanes on 4 neighbouring bins (cp.async, double-buffered over
// batches of k1), and the SPEC outputs are collected in the row buffers and
// written 8 rows x 1 k1 per 8 lanes.
// ----------------------------------------------------------------------------
enum { PAIR = 0, SELF0 = 1, SELFH = 2 };

__host__ __device__ constexpr int rp_batches(int log_n1) { return (1 << log_n1) / 64 >= 4 ? 4 : (1 << log_n1) / 64; }
// Staging rows are BK + 2 complex apart: the four lanes that copy the bins of
// four neighbouring rows at one k1 then land 8 banks apart instead of on
// one bank (the cp.async writes were 96% of the pass's bank conflicts).
__host__ __device__ constexpr int rp_stage_stride(int log_n1) {
    return (1 << log_n1) / 2 / rp_batches(log_n1) + 2;
}

__device__ __forceinline__ void cpa8(void *smem, const void *g) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(g) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int LOG_N1, bool SPEC>
__host__ __device__ constexpr size_t rowpass_smem_bytes() {
    // row buffers, then (conv) two staging buffers of [8 rows][k, M-k][N1/2 / batches + 2]
    return sizeof(float2) * ((size_t)WARPS * spad_size(1 << LOG_N1) +
                             (SPEC ? 0 : (size_t)2 * WARPS * 2 * rp_stage_stride(LOG_N1)));
}

template <int LOG_N1, int LOG_N2, bool SPEC>
__global__ void __launch_bounds__(NT, 2) rowpass_kernel(const FsParams p) {
    constexpr int N1 = 1 << LOG_N1;
    constexpr int N2 = 1 << LOG_N2;
    constexpr int M = N1 * N2;
    constexpr int LP = fs_log_p(LOG_N1);
    constexpr int P = 1 << LP;
    constexpr int RS = spad_size(N1);
    constexpr int NB = rp_batches(LOG_N1);    // staging batches over the owned k1 < N1/2
    constexpr int MB = P / 2 / NB;            // m values per batch
    constexpr int BK = 32 * MB;               // k1 values per batch
    constexpr int HS = rp_stage_stride(LOG_N1);   // staging row stride (BK + 2)
    static_assert(NB >= 1 && MB >= 1 && MB * NB * 2 == P, "row pass batching");
    extern __shared__ float2 rows_s[];        // WARPS rows x RS, then the staging buffers
    float2 *hstage = rows_s + WARPS * RS;     // [2 buffers][8 rows][k, M-k][HS]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x;
    const int64_t row = p.row0 + blockIdx.y;
    const int64_t rl = blockIdx.y;
    float2 *buf = p.buf + rl * (int64_t)M;

    // row of warp w (w < 4: low rows, w >= 4: their mirrors)
    auto row_k2 = [&](int w) {
        if (w < 4) return 4 * g + w;
        return (g == 0 && w == 4) ? N2 / 2 : N2 - (4 * g + w - 4);
    };
    const int k2 = row_k2(warp);
    const int mode = (g == 0 && warp == 0) ? SELF0 : ((g == 0 && warp == 4) ? SELFH : PAIR);
    const int partner = mode == PAIR ? (warp ^ 4) : warp;
    float2 *own = rows_s + warp * RS;
    float2 *oth = rows_s + partner * RS;

    const int64_t d = row % p.D;
    const float2 *H = SPEC ? nullptr : p.spec + d * (int64_t)(M + 1);
    const float dk = (!SPEC && p.skip_k) ? __ldg(p.skip_k + d) : 0.f;   // skip term: H_k + D_k
    float2 *Ho = SPEC ? p.Hout + row * (int64_t)(M + 1) : nullptr;

    // staging of batch b: [w][0][kk] = H[k], [w][1][kk] = H[M - k] with
    // k = k2_w + N2 (b BK + kk); thread: rows j and 4 + j, kk = tid/4 + 64 i
    const int sj = tid & 3, skk = tid >> 2;
    const uint32_t k_lo = (uint32_t)row_k2(sj) + (uint32_t)N2 * (uint32_t)skk;
    const uint32_t k_hi = (uint32_t)row_k2(4 + sj) + (uint32_t)N2 * (uint32_t)skk;
    auto stage = [&](int b, float2 *dst) {
#pragma unroll
        for (int i = 0; i < (BK + NT / 4 - 1) / (NT / 4); ++i) {
            const int kk = skk + i * (NT / 4);
            if (kk < BK) {
                const uint32_t off = (uint32_t)N2 * (uint32_t)(b * BK + i * (NT / 4));
                cpa8(dst + (2 * sj + 0) * HS + kk, H + (k_lo + off));
                cpa8(dst + (2 * sj + 1) * HS + kk, H + (M - (k_lo + off)));
                cpa8(dst + (2 * (4 + sj) + 0) * HS + kk, H + (k_hi + off));
                cpa8(dst + (2 * (4 + sj) + 1) * HS + kk, H + (M - (k_hi + off)));
            }
        }
    };
    if constexpr (!SPEC) {
        stage(0, hstage);
        cpa_commit();
    }

    // ---- load the row (contiguous) and forward FFT over n1 -> bins k2 + N2 k1
    float2 x[P];
    const float2 *src = buf + (int64_t)N1 * k2;
#pragma unroll
    for (int m = 0; m < P; ++m) x[m] = __ldcg(src + lane + 32 * m);
    block_fft<LOG_N1, LP, -1, false, SyncWarp>(x, own, lane, p.tw_n1, SyncWarp{});
#pragma unroll
    for (int m = 0; m < P; ++m) own[spad(lane + 32 * m)] = x[m];
    __syncthreads();

    // ---- pairs of the owned bins k1 = lane + 32 m < N1/2 (m < P/2);
    //      W_{2M}^{k2 + N2 k1} = W_{2M}^{k2 + N2 lane} W_{2M}^{32 N2 m}
    const float2 wl = tw2(p.tw_2m, p.lo_2m, (uint32_t)k2 + (uint32_t)N2 * (uint32_t)lane);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const float2 *hs = hstage + (b & 1) * (WARPS * 2 * HS);
        if constexpr (!SPEC) {
            if (b + 1 < NB) {
                stage(b + 1, hstage + ((b + 1) & 1) * (WARPS * 2 * HS));
                cpa_commit();
                cpa_wait<1>();
            } else {
                cpa_wait<0>();
            }
            __syncthreads();
        }
#pragma unroll
        for (int mm = 0; mm < MB; ++mm) {
            const int m = b * MB + mm;
            const int k1 = lane + 32 * m;
            const int pk1 = mode == SELF0 ? ((N1 - k1) & (N1 - 1)) : (N1 - 1 - k1);
            const float2 zk = x[m];
            float2 hk = make_float2(0.f, 0.f), hn = make_float2(0.f, 0.f);
            if constexpr (!SPEC) {
                hk = hs[(2 * warp + 0) * HS + lane + 32 * mm];
                hn = hs[(2 * warp + 1) * HS + lane + 32 * mm];
                hk.x += dk;
                hn.x += dk;
            }
            if (mode == SELF0 && k1 == 0) {
                // DC (bin 0) and Nyquist (bin M): both real
                if constexpr (SPEC) {
                    own[spad(0)] = make_float2(zk.x + zk.y, 0.f);
                    Ho[M] = make_float2(zk.x - zk.y, 0.f);
                } else {
                    const float y0 = 2.f * (zk.x + zk.y) * hk.x;
                    const float yM = 2.f * (zk.x - zk.y) * hn.x;
                    x[m] = make_float2(y0 + yM, y0 - yM);
                }
                continue;
            }
            const float2 zn = oth[spad(pk1)];
            const float2 A = make_float2(zk.x + zn.x, zk.y - zn.y);
            const float2 Bv = make_float2(zk.x - zn.x, zk.y + zn.y);
            const float2 w = cmul(wl, tw2(p.tw_2m, p.lo_2m, 32u * (uint32_t)N2 * (uint32_t)m));   // W_{2M}^k
            const float2 wB = cmul(Bv, w);
            const float2 C = make_float2(wB.y, -wB.x);
            const float2 Xk = cadd(A, C);                                 // 2 X[k]
            const float2 Xn = cconj(csub(A, C));                          // 2 X[M-k]
            if constexpr (SPEC) {
                own[spad(k1)] = make_float2(0.5f * Xk.x, 0.5f * Xk.y);
                oth[spad(pk1)] = make_float2(0.5f * Xn.x, 0.5f * Xn.y);
            } else {
                const float2 Yk = cmul(Xk, hk);
                const float2 Yn = cmul(Xn, hn);
                const float2 A2 = make_float2(Yk.x + Yn.x, Yk.y - Yn.y);
                const float2 B2 = make_float2(Yk.x - Yn.x, Yk.y + Yn.y);
                const float2 cB = cmulc(B2, w);
                const float2 C2 = make_float2(-cB.y, cB.x);
                x[m] = cadd(A2, C2);
                oth[spad(pk1)] = cconj(csub(A2, C2));
            }
        }
        if constexpr (!SPEC) __syncthreads();   // staging buffer b & 1 is refilled next
    }
    if constexpr (SPEC) {
        // bin M/2 (row 0, k1 = N1/2) pairs with itself: X[M/2] = conj(Z[M/2])
        if (mode == SELF0 && lane == 0) own[spad(N1 / 2)] = cconj(x[(N1 / 2) / 32]);
        __syncthreads();
        // rows_s[w][k1] now holds bin k2_w + N2 k1 of every row of the CTA;
        // 8 lanes store the 8 rows' bins of one k1
        const int w = tid & 7;
        const int kw = row_k2(w);
#pragma unroll 4
        for (int k1 = tid >> 3; k1 < N1; k1 += NT / 8)
            Ho[(uint32_t)kw + (uint32_t)N2 * (uint32_t)k1] = rows_s[w * RS + spad(k1)];
        return;
    }
    // self-paired element of row 0: bin M/2 (k1 = N1/2)
    if (mode == SELF0 && lane == 0) {
        constexpr int mh = (N1 / 2) / 32;
        float2 hm = __ldg(H + M / 2);
        hm.x += dk;
        const float2 r = cmulc(x[mh], hm);
        x[mh] = make_float2(4.f * r.x, 4.f * r.y);
    }
    __syncthreads();
    // bins k1 >= N1/2 were produced by the partner warp (or this one)
#pragma unroll
    for (int m = P / 2; m < P; ++m) {
        const int k1 = lane + 32 * m;
        if (!(mode == SELF0 && k1 == N1 / 2)) x[m] = own[spad(k1)];
    }
    __syncwarp();
    // ---- inverse FFT over k1 -> n1, times W_M^{-n1 k2}, back to the buffer
    block_fft<LOG_N1, LP, +1, false, SyncWarp>(x, own, lane, p.tw_n1, SyncWarp{});
    float2 *dst = buf + (int64_t)N1 * k2;
    const float2 tl = tw2(p.tw_m, p.lo_m, ((uint32_t)k2 * (uint32_t)lane) & (M - 1));
#pragma unroll
    for (int m = 0; m < P; ++m) {
        const float2 t = cmul(tl, tw2(p.tw_m, p.lo_m, (32u * (uint32_t)k2 * (uint32_t)m) & (M - 1)));
        __stcg(dst + lane + 32 * m, cmulc(x[m], t));
    }
}

// Rows per chunk: the complex buffer of a chunk (8 bytes per point) is kept
// near 104 MB.  At M = 2^20, 64 and 96 MB chunks measured the same and 32 MB
// ones slower, although only the smaller chunks keep the buffer in L2 between
// passes: the passes are latency-bound, and short launches lose to their tail.
// 104 MB is 13 rows there (1664 CTAs per pass: 3.75 waves of the column
// passes' three CTAs per SM, 5.6 of the row pass's two), 1.6% faster than 12.
int64_t chunk_rows_of(int64_t rows, int log_mc) {
    const int64_t per_row = (int64_t)8 << log_mc;
    int64_t c = ((int64_t)104 << 20) / per_row;
    if (c < 1) c = 1;
    return c < rows ? c : rows;
}


// Every row start of u, the gates and y is aligned for 4-element vectors.
bool vec4_rows(const LongConvArgs &a, size_t el) {
    const uintptr_t al = 4 * el;
    if (a.L % 4 != 0 || (uintptr_t)a.u % al || (uintptr_t)a.y % al) return false;
    for (int k = 0; k < a.K; ++k)
        if (a.gate[k] && (uintptr_t)a.gate[k] % al) return false;
    return true;
}

template <typename Kern>
hy_status smem_attr(Kern k, size_t bytes) {
    if (bytes > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return set_cuda_error("multi-pass smem attribute", e);
    }
    // the column passes run three CTAs per SM: all of shared memory is asked for
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return set_cuda_error("multi-pass carveout attribute", e);
    return HY_OK;
}

// Tensor map of fp32 input rows of exactly M = N1 N2 samples seen as a 2-D
// array of rows x N2/2 rows of 2 N1 floats (pass A's input tiles); p->in_tma
// says whether it applies (length, 16-byte alignment).
hy_status input_map(CUtensorMap *m, int *in_tma, const void *in, int64_t rows, int64_t L, int log_n1, int log_n2) {
    const uint64_t n1 = (uint64_t)1 << log_n1, n2 = (uint64_t)1 << log_n2;
    *in_tma = 0;
    memset(m, 0, sizeof(*m));
    if (L != (int64_t)(n1 * n2) || ((uintptr_t)in & 15) != 0) return HY_OK;
    const uint64_t half = n2 / 2;
    hy_status st = tma_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, in, 2 * n1, (uint64_t)rows * half, 8 * n1, 16,
                              (uint32_t)(half < (uint64_t)kTileBoxRows ? half : (uint64_t)kTileBoxRows),
                              CU_TENSOR_MAP_SWIZZLE_64B, "multi-pass input tiles");
    if (st == HY_OK) *in_tma = 1;
    return st;
}

// Tensor map of the chunk's complex buffer as a 2-D fp32 array: rows_chunk x
// N2 rows of 2 N1 floats (row pitch 8 N1 bytes), boxes of 16 floats (8
// complex columns, 64 bytes) x min(N2, 256) rows, 64-byte swizzle.
hy_status buf_map(CUtensorMap *m, const float2 *buf, int log_n1, int log_n2, int64_t rows_chunk) {
    const uint64_t n1 = (uint64_t)1 << log_n1, n2 = (uint64_t)1 << log_n2;
    return tma_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, buf, 2 * n1, (uint64_t)rows_chunk * n2, 8 * n1, 16,
                      (uint32_t)(n2 < (uint64_t)kTileBoxRows ? n2 : (uint64_t)kTileBoxRows),
                      CU_TENSOR_MAP_SWIZZLE_64B, "multi-pass column tiles");
}

template <int LOG_N1, int LOG_N2, typename IO>
hy_status run_conv(const LongConvArgs &a, cudaStream_t s) {
    constexpr int N1 = 1 << LOG_N1, N2 = 1 << LOG_N2;
    constexpr int LOG_MC = LOG_N1 + LOG_N2;
    const int64_t rows = a.B * a.D;
    const int64_t cr = chunk_rows_of(rows, LOG_MC);
    FsParams p{};
    p.D = a.D;
    p.L = (int)a.L;
    p.K = a.K;
    p.u = a.u;
    p.y = a.y;
    p.buf = reinterpret_cast<float2 *>(a.ws);
    p.scale = (float)(1.0 / (4.0 * (double)((int64_t)1 << LOG_MC)));
    p.vec4 = vec4_rows(a, sizeof(IO));
    p.tw_n1 = tw_stages(LOG_N1, fs_log_p(LOG_N1));
    p.tw_n2 = tw_stages(LOG_N2, fs_log_p(LOG_N2));
    p.lo_m = LOG_MC / 2;
    p.tw_m = tw_pow2(LOG_MC, p.lo_m);
    p.lo_2m = (LOG_MC + 1) / 2;
    p.tw_2m = tw_pow2(LOG_MC + 1, p.lo_2m);
    if (!p.tw_n1 || !p.tw_n2 || !p.tw_m || !p.tw_2m) return set_error(HY_ERR_CUDA, "multi-pass twiddle tables missing");
    p.fault = device_fault_word();
    const size_t chunk_el = (size_t)cr << LOG_MC;           // complex points of one chunk buffer
    const int want = chunk_lanes(rows, cr, (size_t)8 << LOG_MC, a.ws_bytes);
    float2 *bufs[kMaxLanes];
    CUtensorMap bmap[kMaxLanes], imap;
    hy_status st;
    for (int l = 0; l < want; ++l) {
        bufs[l] = p.buf + (size_t)l * chunk_el;
        if ((st = buf_map(&bmap[l], bufs[l], LOG_N1, LOG_N2, cr)) != HY_OK) return st;
    }
    // gates of the pass C epilogues: same geometry as the input, prefetched into L2
    CUtensorMap gmap[8];
    int gpf[8] = {0};
    if (sizeof(IO) == 4) {
        if ((st = input_map(&imap, &p.in_tma, a.u, rows, a.L, LOG_N1, LOG_N2)) != HY_OK) return st;
        for (int k = 0; k < a.K; ++k) {
            memset(&gmap[k], 0, sizeof(gmap[k]));
            if (a.gate[k] && (st = input_map(&gmap[k], &gpf[k], a.gate[k], rows, a.L, LOG_N1, LOG_N2)) != HY_OK)
                return st;
        }
    } else {
        memset(&imap, 0, sizeof(imap));
        p.in_tma = 0;
        for (int k = 0; k < a.K; ++k) memset(&gmap[k], 0, sizeof(gmap[k]));
    }
    p.gate_pf = 0;
    const size_t smem_c = colpass_smem_bytes<LOG_N2>();
    const size_t smem_r = rowpass_smem_bytes<LOG_N1, false>();
    auto kA = colpass_kernel<LOG_N1, LOG_N2, IO, false, true, false>;
    auto kCA = colpass_kernel<LOG_N1, LOG_N2, IO, true, true, false>;
    auto kC = colpass_kernel<LOG_N1, LOG_N2, IO, true, false, false>;
    auto kB = rowpass_kernel<LOG_N1, LOG_N2, false>;
    if ((st = smem_attr(kA, smem_c)) != HY_OK || (st = smem_attr(kCA, smem_c)) != HY_OK ||
        (st = smem_attr(kC, smem_c)) != HY_OK || (st = smem_attr(kB, smem_r)) != HY_OK)
        return st;
    LaneScope lanes;
    if ((st = lanes.open(want, s)) != HY_OK) return st;
    int ci = 0;
    for (int64_t r0 = 0; r0 < rows; r0 += cr, ++ci) {
        const int64_t nr = (rows - r0) < cr ? (rows - r0) : cr;
        const int ln = lanes.lane_of(ci);
        const cudaStream_t cs = lanes.stream_of(ci);
        p.buf = bufs[ln];
        p.row0 = r0;
        dim3 gc(N1 / WARPS, (unsigned)nr), gr(N2 / 8, (unsigned)nr);
        p.k = 0;
        kA<<<gc, NT, smem_c, cs>>>(p, bmap[ln], imap);
        for (int k = 0; k < a.K; ++k) {
            p.k = k;
            p.spec = a.spec[k];
            p.gate_k = a.gate[k];
            p.skip_k = a.skip[k];
            kB<<<gr, NT, smem_r, cs>>>(p);
            p.gate_pf = gpf[k];
            if (k + 1 < a.K) kCA<<<gc, NT, smem_c, cs>>>(p, bmap[ln], gmap[k]);
            else kC<<<gc, NT, smem_c, cs>>>(p, bmap[ln], gmap[k]);
            p.gate_pf = 0;
        }
        if ((st = check_launch("multi-pass conv launch")) != HY_OK) return st;
    }
    return lanes.join();
}

template <int LOG_N1, int LOG_N2>
hy_status run_spectrum(int64_t rows, int64_t L, const float *h, float2 *H, void *ws, size_t ws_bytes,
                       cudaStream_t s) {
    constexpr int N1 = 1 << LOG_N1, N2 = 1 << LOG_N2;
    constexpr int LOG_MC = LOG_N1 + LOG_N2;
    const int64_t cr = chunk_rows_of(rows, LOG_MC);
    FsParams p{};
    p.D = 1;
    p.L = (int)L;
    p.K = 1;
    p.u = h;
    p.buf = reinterpret_cast<float2 *>(ws);
    p.Hout = H;
    p.vec4 = L % 4 == 0 && (uintptr_t)h % 16 == 0;
    p.tw_n1 = tw_stages(LOG_N1, fs_log_p(LOG_N1));
    p.tw_n2 = tw_stages(LOG_N2, fs_log_p(LOG_N2));
    p.lo_m = LOG_MC / 2;
    p.tw_m = tw_pow2(LOG_MC, p.lo_m);
    p.lo_2m = (LOG_MC + 1) / 2;
    p.tw_2m = tw_pow2(LOG_MC + 1, p.lo_2m);
    if (!p.tw_n1 || !p.tw_n2 || !p.tw_m || !p.tw_2m) return set_error(HY_ERR_CUDA, "multi-pass twiddle tables missing");
    p.fault = device_fault_word();
    const size_t chunk_el = (size_t)cr << LOG_MC;
    const int want = chunk_lanes(rows, cr, (size_t)8 << LOG_MC, ws_bytes);
    float2 *bufs[kMaxLanes];
    CUtensorMap bmap[kMaxLanes], imap;
    hy_status st;
    for (int l = 0; l < want; ++l) {
        bufs[l] = p.buf + (size_t)l * chunk_el;
        if ((st = buf_map(&bmap[l], bufs[l], LOG_N1, LOG_N2, cr)) != HY_OK) return st;
    }
    if ((st = input_map(&imap, &p.in_tma, h, rows, L, LOG_N1, LOG_N2)) != HY_OK) return st;
    const size_t smem_c = colpass_smem_bytes<LOG_N2>();
    const size_t smem_r = rowpass_smem_bytes<LOG_N1, true>();
    auto kA = colpass_kernel<LOG_N1, LOG_N2, float, false, true, true>;
    auto kB = rowpass_kernel<LOG_N1, LOG_N2, true>;
    if ((st = smem_attr(kA, smem_c)) != HY_OK || (st = smem_attr(kB, smem_r)) != HY_OK) return st;
    LaneScope lanes;
    if ((st = lanes.open(want, s)) != HY_OK) return st;
    int ci = 0;
    for (int64_t r0 = 0; r0 < rows; r0 += cr, ++ci) {
        const int64_t nr = (rows - r0) < cr ? (rows - r0) : cr;
        const int ln = lanes.lane_of(ci);
        const cudaStream_t cs = lanes.stream_of(ci);
        p.buf = bufs[ln];
        p.row0 = r0;
        kA<<<dim3(N1 / WARPS, (unsigned)nr), NT, smem_c, cs>>>(p, bmap[ln], imap);
        kB<<<dim3(N2 / 8, (unsigned)nr), NT, smem_r, cs>>>(p);
        if ((st = check_launch("multi-pass spectrum launch")) != HY_OK) return st;
    }
    return lanes.join();
}

}  // namespace

// The device's second stream and events for the chunk pipelines
// (chunk_lanes.h), made on first use and kept for the process.
ChunkLanes *chunk_lanes_of_device() {
    constexpr int kMaxDevices = 64;
    static ChunkLanes lanes[kMaxDevices];
    static std::once_flag once[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    ChunkLanes *l = &lanes[dev];
    static bool ok[kMaxDevices];
    std::call_once(once[dev], [l, dev] {
        bool good = cudaEventCreateWithFlags(&l->fork, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; good && i + 1 < kMaxLanes; ++i)
            good = cudaStreamCreateWithFlags(&l->extra[i], cudaStreamNonBlocking) == cudaSuccess &&
                   cudaEventCreateWithFlags(&l->join[i], cudaEventDisableTiming) == cudaSuccess;
        if (!good) cudaGetLastError();
        ok[dev] = good;
    });
    return ok[dev] ? l : nullptr;
}

// Workspace: one chunk buffer at least; the queries return one per lane
// that can be busy (chunk_lanes.h).
size_t long_workspace_of(int64_t rows, int log_mc, bool minimum) {
    if (log_mc < 15 || log_mc > 20) return 0;
    const int64_t cr = chunk_rows_of(rows, log_mc);
    return minimum ? (size_t)cr * ((size_t)8 << log_mc) : chunk_workspace(rows, cr, (size_t)8 << log_mc);
}

size_t long_conv_workspace(int64_t B, int64_t D, int log_mc, int) { return long_workspace_of(B * D, log_mc, false); }
size_t long_conv_workspace_min(int64_t B, int64_t D, int log_mc) { return long_workspace_of(B * D, log_mc, true); }
size_t long_spectrum_workspace(int64_t rows, int log_mc) { return long_workspace_of(rows, log_mc, false); }
size_t long_spectrum_workspace_min(int64_t rows, int log_mc) { return long_workspace_of(rows, log_mc, true); }

hy_status launch_long_conv(const LongConvArgs &a, cudaStream_t s) {
    const bool bf = a.dt == HY_BF16;
    switch (a.log_mc) {
#define HY_LC(LM, N1L, N2L) \
    case LM: return bf ? run_conv<N1L, N2L, __nv_bfloat16>(a, s) : run_conv<N1L, N2L, float>(a, s);
        HY_LC(15, 7, 8) HY_LC(16, 8, 8) HY_LC(17, 8, 9) HY_LC(18, 9, 9) HY_LC(19, 9, 10) HY_LC(20, 10, 10)
#undef HY_LC
        default: return set_error(HY_ERR_UNSUPPORTED, "multi-pass length 2^%d not built", a.log_mc);
    }
}

hy_status launch_long_spectrum(int64_t rows, int64_t L, int log_mc, const float *h, float2 *H, void *ws,
                               size_t ws_bytes, cudaStream_t s) {
    switch (log_mc) {
#define HY_LS(LM, N1L, N2L) \
    case LM: return run_spectrum<N1L, N2L>(rows, L, h, H, ws, ws_bytes, s);
        HY_LS(15, 7, 8) HY_LS(16, 8, 8) HY_LS(17, 8, 9) HY_LS(18, 9, 9) HY_LS(19, 9, 10) HY_LS(20, 10, 10)
#undef HY_LS
        default: return set_error(HY_ERR_UNSUPPORTED, "multi-pass length 2^%d not built", log_mc);
    }
}

}  // namespace hy

// ============================================================================
// Allocation-free variant of the multi-pass operator.
//
// Some callers cannot call cudaMalloc at all: code running inside a custom
// allocator or a memory-pool callback, plugins whose host framework owns every
// device allocation, and real-time loops that must not touch the driver's
// allocator.  For them the multi-pass workspace lives in a fixed static device
// array instead of a caller buffer.  Rows are processed in chunks sized to
// that array, with the same kernels as launch_long_conv.
// ============================================================================
namespace hy {

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)32 << 20;   // 32 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {nullptr};

// Device address of the scratch array for the current device.  Host code
// cannot use the array's name as a device address; it is resolved once per
// device with cudaGetSymbolAddress while that device is current.
hy_status noalloc_scratch(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return set_error(HY_ERR_UNSUPPORTED, "device index %d >= 64", dev);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return set_cuda_error("cudaGetSymbolAddress(no-alloc scratch)", e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return HY_OK;
}

template <int LOG_N1, int LOG_N2, typename IO>
hy_status run_conv_static(const LongConvArgs &a, void *scratch, cudaStream_t s) {
    constexpr int N1 = 1 << LOG_N1, N2 = 1 << LOG_N2;
    constexpr int LOG_MC = LOG_N1 + LOG_N2;
    const int64_t rows = a.B * a.D;
    const size_t per_row = (size_t)8 << LOG_MC;
    int64_t cr = (int64_t)(kNoAllocScratchBytes / per_row);
    if (cr < 1)
        return set_error(HY_ERR_WORKSPACE, "hyena_operator_noalloc: one row needs %zu bytes, the static scratch holds %zu",
                         per_row, kNoAllocScratchBytes);
    if (cr > rows) cr = rows;
    FsParams p{};
    p.D = a.D;
    p.L = (int)a.L;
    p.K = a.K;
    p.u = a.u;
    p.y = a.y;
    p.buf = reinterpret_cast<float2 *>(scratch);
    p.scale = (float)(1.0 / (4.0 * (double)((int64_t)1 << LOG_MC)));
    p.vec4 = vec4_rows(a, sizeof(IO));
    p.tw_n1 = tw_stages(LOG_N1, fs_log_p(LOG_N1));
    p.tw_n2 = tw_stages(LOG_N2, fs_log_p(LOG_N2));
    p.lo_m = LOG_MC / 2;
    p.tw_m = tw_pow2(LOG_MC, p.lo_m);
    p.lo_2m = (LOG_MC + 1) / 2;
    p.tw_2m = tw_pow2(LOG_MC + 1, p.lo_2m);
    if (!p.tw_n1 || !p.tw_n2 || !p.tw_m || !p.tw_2m) return set_error(HY_ERR_CUDA, "multi-pass twiddle tables missing");
    p.fault = device_fault_word();
    CUtensorMap bmap, imap;
    hy_status st = buf_map(&bmap, p.buf, LOG_N1, LOG_N2, cr);
    if (st != HY_OK) return st;
    // gates of the pass C epilogues: same geometry as the input, prefetched into L2
    CUtensorMap gmap[8];
    int gpf[8] = {0};
    if (sizeof(IO) == 4) {
        if ((st = input_map(&imap, &p.in_tma, a.u, rows, a.L, LOG_N1, LOG_N2)) != HY_OK) return st;
        for (int k = 0; k < a.K; ++k) {
            memset(&gmap[k], 0, sizeof(gmap[k]));
            if (a.gate[k] && (st = input_map(&gmap[k], &gpf[k], a.gate[k], rows, a.L, LOG_N1, LOG_N2)) != HY_OK)
                return st;
        }
    } else {
        memset(&imap, 0, sizeof(imap));
        p.in_tma = 0;
        for (int k = 0; k < a.K; ++k) memset(&gmap[k], 0, sizeof(gmap[k]));
    }
    p.gate_pf = 0;
    const size_t smem_c = colpass_smem_bytes<LOG_N2>();
    const size_t smem_r = rowpass_smem_bytes<LOG_N1, false>();
    auto kA = colpass_kernel<LOG_N1, LOG_N2, IO, false, true, false>;
    auto kCA = colpass_kernel<LOG_N1, LOG_N2, IO, true, true, false>;
    auto kC = colpass_kernel<LOG_N1, LOG_N2, IO, true, false, false>;
    auto kB = rowpass_kernel<LOG_N1, LOG_N2, false>;
    if ((st = smem_attr(kA, smem_c)) != HY_OK || (st = smem_attr(kCA, smem_c)) != HY_OK ||
        (st = smem_attr(kC, smem_c)) != HY_OK || (st = smem_attr(kB, smem_r)) != HY_OK)
        return st;
    // Nothing in the scratch has to start at zero: pass A writes every complex
    // point of a row before pass B reads it.
    for (int64_t r0 = 0; r0 < rows; r0 += cr) {
        const int64_t nr = (rows - r0) < cr ? (rows - r0) : cr;
        p.row0 = r0;
        dim3 gc(N1 / WARPS, (unsigned)nr), gr(N2 / 8, (unsigned)nr);
        p.k = 0;
        kA<<<gc, NT, smem_c, s>>>(p, bmap, imap);
        for (int k = 0; k < a.K; ++k) {
            p.k = k;
            p.spec = a.spec[k];
            p.gate_k = a.gate[k];
            p.skip_k = a.skip[k];
            kB<<<gr, NT, smem_r, s>>>(p);
            p.gate_pf = gpf[k];
            if (k + 1 < a.K) kCA<<<gc, NT, smem_c, s>>>(p, bmap, gmap[k]);
            else kC<<<gc, NT, smem_c, s>>>(p, bmap, gmap[k]);
            p.gate_pf = 0;
        }
        if ((st = check_launch("no-alloc multi-pass launch")) != HY_OK) return st;
    }
    return HY_OK;
}

}  // namespace

size_t noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

hy_status launch_long_conv_noalloc(const LongConvArgs &a, cudaStream_t s) {
    void *scratch = nullptr;
    hy_status st = noalloc_scratch(&scratch);
    if (st != HY_OK) return st;
    const bool bf = a.dt == HY_BF16;
    switch (a.log_mc) {
#define HY_LC(LM, N1L, N2L) \
    case LM: return bf ? run_conv_static<N1L, N2L, __nv_bfloat16>(a, scratch, s) : run_conv_static<N1L, N2L, float>(a, scratch, s);
        HY_LC(15, 7, 8) HY_LC(16, 8, 8) HY_LC(17, 8, 9) HY_LC(18, 9, 9) HY_LC(19, 9, 10) HY_LC(20, 10, 10)
#undef HY_LC
        default: return set_error(HY_ERR_UNSUPPORTED, "hyena_operator_noalloc: length 2^%d beyond the static scratch", a.log_mc);
    }
}

}  // namespace hy
