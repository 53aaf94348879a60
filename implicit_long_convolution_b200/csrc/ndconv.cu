// ndconv.cu -- HyenaND global 3-D convolution with gating and 3-D filter
// spectra ([ND] 방법론: HyenaND -- 네이티브 ND 합성곱 through the N-D FFT; 경계
// 처리: circular, or non-circular by zero-padding every axis to double).
//
// A slab (one sample, one channel) of g^3 samples is transformed on the cube
// of edge S (S = 2g non-circular, S = g circular), separably:
//   F1 (one CTA per x-plane i):  real FFT along z of each y-row (packed into
//       S/2 complex points, split into S/2+1 bins), then FFT along y of each
//       bin column; the plane (S x (S/2+1)) goes to the workspace.
//   F2 (one CTA per y-bin k1):   FFT along x of each (k1, kz) line, times the
//       kernel spectrum H[kx, k1, kz], inverse FFT along x (conv), or the
//       spectrum itself written out (filter spectrum).
//   F3 (one CTA per x-plane i):  inverse FFT along y, then the inverse real
//       FFT along z of each row (merge + packed inverse), crop to the grid,
//       skip term and gate, output.
// Zero-padded halves are never read (the first butterfly stage of a padded
// axis skips them) and cropped halves are never written.  Each small FFT is
// done by a group of S/16 or S/32 threads (8 points per thread) with warp
// synchronisation; planes stay in shared memory; slabs are processed in
// chunks whose workspace stays in L2 between the passes.
#include "chunk_lanes.h"
#include "kernels.h"
#include "fft_core.cuh"
#include "status.h"
#include "twiddle.h"

namespace hy {

namespace {

constexpr int NT = 256;

__host__ __device__ constexpr int nd_log_p(int log_n) { return log_n < 3 ? log_n : 3; }
// The column transforms of the plane kernels (F1, F3) at 128 points take 16
// points per thread: one exchange instead of two (the x pass keeps 8, its
// staging of the kernel spectrum would not fit beside the wider groups).
__host__ __device__ constexpr int nd_col_log_p(int log_n) { return log_n >= 7 ? 4 : nd_log_p(log_n); }

struct NdParams {
    int64_t slab0;              // first slab of the chunk (b*D + d)
    int64_t D;
    const float *u;             // conv: (B, D, g, g, g); spectrum: rows of S^3
    const float *gate;
    const float *skip;
    const float2 *H;            // conv: kernel spectra; spectrum: output
    int64_t H_batch_stride;     // complex elements between samples (0 = shared)
    float2 *Hout;
    float2 *ws;                 // chunk_slabs x gI x S x (S/2+1)
    float *y;
    float scale;
    const float2 *tw_r;         // row FFT (S/2 points) stage tables
    const float2 *tw_c;         // column FFT (S points) stage tables
    const float2 *tw_cp;        // the plane kernels' column FFT (nd_col_log_p) stage tables
    const float2 *tw_split;     // W_S^k, k <= S/4
};

// W_S^k for 0 <= k < S/2 from the table of k <= S/4 (W^k = -conj W^{S/2-k})
__device__ __forceinline__ float2 wsplit(const float2 *tab, int k, int half) {
    if (2 * k <= half) return __ldg(tab + k);
    const float2 w = __ldg(tab + (half - k));
    return make_float2(-w.x, w.y);
}

// One small FFT per group of T = N/P threads; group g, lane t within group.
// Its exchange buffer pads one slot every 2^SH elements and groups follow
// each other every N + N/2^SH slots: with several groups in a warp this makes
// the stride-8 writes of the first stage and the reads back conflict-free
// (up to 64 points) or nearly so (128).
template <int LOG_N, int LOG_P = nd_log_p(LOG_N)>
struct Grp {
    static constexpr int N = 1 << LOG_N;
    static constexpr int LP = LOG_P;
    static constexpr int P = 1 << LP;
    static constexpr int T = N / P;
    static constexpr int G = NT / T;
    static constexpr int SH = LOG_N <= 6 ? 3 : 4;
    static constexpr int BUF = N + (N >> SH);       // exchange buffer of a group
};

// ---------------------------------------------------------------------------
// F1: forward along z (real) and y for one x-plane.
// ---------------------------------------------------------------------------
template <int LOG_S, bool PAD>
__global__ void __launch_bounds__(NT) nd_fwd_plane(const NdParams p) {
    constexpr int S = 1 << LOG_S;
    constexpr int H2 = S / 2;               // packed row length = real bins - 1
    constexpr int NB = H2 + 1;              // bins along z
    constexpr int gI = PAD ? S / 2 : S;     // input extent per axis
    using R = Grp<LOG_S - 1>;               // row FFT, H2 points
    using C = Grp<LOG_S>;                   // column FFT, S points
    extern __shared__ float2 sm[];
    float2 *tile = sm;                                  // S rows x NB (row j, bin k)
    float2 *gbuf = sm + S * NB;                         // group exchange buffers
    const int tid = threadIdx.x;
    const int64_t slab = p.slab0 + blockIdx.y;
    const int i = blockIdx.x;                           // x-plane
    const float *plane = p.u + (slab * gI + i) * (int64_t)gI * gI;

    constexpr int PK = gI / 2;                          // packed points per row

    // ---- row pass: real FFT along z of rows j < gI
    {
        const int g = tid / R::T, t = tid % R::T;
        float2 *xb = gbuf + g * R::BUF;
        // the next round's row is requested before this round's FFT
        auto load_row = [&](int j, float2 (&v)[R::P]) {
#pragma unroll
            for (int m = 0; m < R::P; ++m) {
                const int e = t + m * R::T;             // packed point
                v[m] = make_float2(0.f, 0.f);
                if (j < gI && e < PK) v[m] = __ldg(reinterpret_cast<const float2 *>(plane + (int64_t)j * gI) + e);
            }
        };
        float2 xn[R::P];
        load_row(g, xn);
        for (int j0 = 0; j0 < gI; j0 += R::G) {
            const int j = j0 + g;
            const bool act = j < gI;
            float2 x[R::P];
#pragma unroll
            for (int m = 0; m < R::P; ++m) x[m] = xn[m];
            if (j0 + R::G < gI) load_row(j + R::G, xn);
            block_fft<LOG_S - 1, R::LP, -1, PAD, SyncWarp, R::SH>(x, xb, t, p.tw_r, SyncWarp{});
            store_own<LOG_S - 1, R::LP, R::SH>(x, xb, t);
            __syncwarp();
            // split: bins k = t + m*T (k < H2) and the Nyquist bin H2
#pragma unroll
            for (int m = 0; m < R::P; ++m) {
                const int k = t + m * R::T;
                const float2 zk = x[m];
                const float2 zn = xb[spadx<R::SH>((H2 - k) & (H2 - 1))];
                const float2 A = make_float2(zk.x + zn.x, zk.y - zn.y);
                const float2 Bv = make_float2(zk.x - zn.x, zk.y + zn.y);
                const float2 wB = cmul(Bv, wsplit(p.tw_split, k, H2));
                const float2 X = make_float2(A.x + wB.y, A.y - wB.x);    // 2 X[k]
                if (act) tile[j * NB + k] = X;
                if (act && k == 0) tile[j * NB + H2] = make_float2(2.f * (zk.x - zk.y), 0.f);
            }
            __syncwarp();
        }
    }
    __syncthreads();
    // ---- column pass: FFT along y of each bin column (inputs j < gI); a
    //      warp whose groups all fall past the last column skips the round
    {
        using CP = Grp<LOG_S, nd_col_log_p(LOG_S)>;
        const int g = tid / CP::T, t = tid % CP::T;
        float2 *xb = gbuf + g * CP::BUF;
        for (int k0 = 0; k0 < NB; k0 += CP::G) {
            if (k0 + (tid >> 5) * (32 / CP::T) >= NB) continue;   // warp-uniform
            const int k = k0 + g;
            const bool act = k < NB;
            float2 x[CP::P];
#pragma unroll
            for (int m = 0; m < CP::P; ++m) {
                const int j = t + m * CP::T;
                x[m] = (act && j < gI) ? tile[j * NB + k] : make_float2(0.f, 0.f);
            }
            block_fft<LOG_S, CP::LP, -1, PAD, SyncWarp, CP::SH>(x, xb, t, p.tw_cp, SyncWarp{});
            __syncwarp();
            if (act) {
#pragma unroll
                for (int m = 0; m < CP::P; ++m) tile[(t + m * CP::T) * NB + k] = x[m];
            }
        }
    }
    __syncthreads();
    // ---- plane out: S x NB complex, contiguous
    float2 *dst = p.ws + ((int64_t)blockIdx.y * gI + i) * (int64_t)S * NB;
    for (int e = tid; e < S * NB; e += NT) __stcg(dst + e, tile[e]);
}

// ---------------------------------------------------------------------------
// F2: along x for one y-bin: conv (times H, inverse, crop) or spectrum out.
// The kernel spectrum H[kx, k1, kz] of this y-bin is S runs of S/2+1
// contiguous bins; each round of G lines (kz) stages its S x G block through
// shared memory (cp.async, two buffers), so HBM sees 128-byte runs instead of
// one 8-byte value per line per kx.  Spectrum outputs go back through the
// tile and leave as contiguous runs.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void nd_cpa8(void *smem, const void *g) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(sa), "l"(g) : "memory");
}
__device__ __forceinline__ void nd_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void nd_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// H staging block of one round: S rows (kx) x G lines, row stride G + 1
template <int LOG_S>
__host__ __device__ constexpr int xpass_hstride() { return Grp<LOG_S>::G + 1; }

template <int LOG_S, bool PAD, bool SPEC>
__global__ void __launch_bounds__(NT) nd_xpass(const NdParams p) {
    constexpr int S = 1 << LOG_S;
    constexpr int H2 = S / 2;
    constexpr int NB = H2 + 1;
    constexpr int gI = PAD ? S / 2 : S;
    using C = Grp<LOG_S>;
    constexpr int G = C::G;                              // lines per round
    constexpr int HS = xpass_hstride<LOG_S>();           // = G + 1
    static_assert(HS == G + 1, "staging stride");
    constexpr int NR = (NB + G - 1) / G;                 // rounds
    extern __shared__ float2 sm[];
    float2 *tile = sm;                                  // gI rows (x) x NB
    float2 *gbuf = sm + gI * NB;
    float2 *hst = gbuf + NT / C::T * C::BUF;   // conv: 2 x [S][HS]
    const int tid = threadIdx.x;
    const int64_t sl = blockIdx.y;                      // slab within chunk
    const int64_t slab = p.slab0 + sl;
    const int k1 = blockIdx.x;
    float2 *base = p.ws + sl * (int64_t)gI * S * NB + (int64_t)k1 * NB;
    for (int e = tid; e < gI * NB; e += NT) {
        const int ii = e / NB, k = e - ii * NB;
        nd_cpa8(tile + e, base + (int64_t)ii * S * NB + k);
    }
    nd_commit();
    const int64_t d = slab % p.D, b = slab / p.D;
    const float2 *Hs = SPEC ? nullptr : p.H + b * p.H_batch_stride + d * (int64_t)S * S * NB + (int64_t)k1 * NB;
    auto stage = [&](int r, float2 *dst) {
        for (int e = tid; e < S * G; e += NT) {
            const int kx = e / G, kk = e % G;
            const int k = r * G + kk;
            if (k < NB) nd_cpa8(dst + kx * HS + kk, Hs + (int64_t)kx * S * NB + k);
        }
    };
    if constexpr (!SPEC) {
        stage(0, hst);
        nd_commit();
    }
    nd_wait<0>();
    __syncthreads();
    const int g = tid / C::T, t = tid % C::T;
    float2 *xb = gbuf + g * C::BUF;
#pragma unroll 1
    for (int r = 0; r < NR; ++r) {
        const int k = r * G + g;
        const bool act = k < NB;
        if constexpr (!SPEC) {
            if (r + 1 < NR) {
                stage(r + 1, hst + ((r + 1) & 1) * S * HS);
                nd_commit();
                nd_wait<1>();
            } else {
                nd_wait<0>();
            }
            __syncthreads();
        }
        float2 x[C::P];
#pragma unroll
        for (int m = 0; m < C::P; ++m) {
            const int ii = t + m * C::T;
            x[m] = (act && ii < gI) ? tile[ii * NB + k] : make_float2(0.f, 0.f);
        }
        block_fft<LOG_S, C::LP, -1, PAD, SyncWarp, C::SH>(x, xb, t, p.tw_c, SyncWarp{});
        if constexpr (SPEC) {
            // back into column k of the tile (gI = S here); the z split
            // carries a factor 2 (folded into the conv scale)
            __syncwarp();
            if (act) {
#pragma unroll
                for (int m = 0; m < C::P; ++m) {
                    const int kx = t + m * C::T;
                    tile[kx * NB + k] = make_float2(0.5f * x[m].x, 0.5f * x[m].y);
                }
            }
        } else {
            const float2 *hb = hst + (r & 1) * S * HS + g;
#pragma unroll
            for (int m = 0; m < C::P; ++m) {
                const int kx = t + m * C::T;
                x[m] = cmul(x[m], act ? hb[kx * HS] : make_float2(0.f, 0.f));
            }
            __syncwarp();
            block_fft<LOG_S, C::LP, +1, false, SyncWarp, C::SH>(x, xb, t, p.tw_c, SyncWarp{});
            __syncwarp();
            if (act) {
#pragma unroll
                for (int m = 0; m < C::P; ++m) {
                    const int ii = t + m * C::T;
                    if (ii < gI) tile[ii * NB + k] = x[m];
                }
            }
            __syncthreads();   // staging buffer r & 1 is refilled next round
        }
    }
    if constexpr (SPEC) {
        __syncthreads();
        float2 *Ho = p.Hout + slab * (int64_t)S * S * NB + (int64_t)k1 * NB;
        for (int e = tid; e < S * NB; e += NT) {
            const int kx = e / NB, k = e - kx * NB;
            Ho[(int64_t)kx * S * NB + k] = tile[e];
        }
    } else {
        for (int e = tid; e < gI * NB; e += NT) {
            const int ii = e / NB, k = e - ii * NB;
            __stcg(base + (int64_t)ii * S * NB + k, tile[e]);
        }
    }
}

// ---------------------------------------------------------------------------
// F3: inverse along y and z (real) for one x-plane, crop, skip, gate, out.
// ---------------------------------------------------------------------------
template <int LOG_S, bool PAD>
__global__ void __launch_bounds__(NT) nd_inv_plane(const NdParams p) {
    constexpr int S = 1 << LOG_S;
    constexpr int H2 = S / 2;
    constexpr int NB = H2 + 1;
    constexpr int gI = PAD ? S / 2 : S;
    using R = Grp<LOG_S - 1>;
    using C = Grp<LOG_S>;
    extern __shared__ float2 sm[];
    float2 *tile = sm;                                  // S rows (k1 -> j) x NB
    float2 *gbuf = sm + S * NB;
    const int tid = threadIdx.x;
    const int64_t sl = blockIdx.y;
    const int64_t slab = p.slab0 + sl;
    const int i = blockIdx.x;
    const float2 *src = p.ws + (sl * gI + i) * (int64_t)S * NB;
    for (int e = tid; e < S * NB; e += NT) nd_cpa8(tile + e, src + e);
    nd_commit();
    nd_wait<0>();
    __syncthreads();
    // ---- inverse along y (k1 -> j), keep j < gI
    {
        using CP = Grp<LOG_S, nd_col_log_p(LOG_S)>;
        const int g = tid / CP::T, t = tid % CP::T;
        float2 *xb = gbuf + g * CP::BUF;
        for (int k0 = 0; k0 < NB; k0 += CP::G) {
            if (k0 + (tid >> 5) * (32 / CP::T) >= NB) continue;   // warp-uniform
            const int k = k0 + g;
            const bool act = k < NB;
            float2 x[CP::P];
#pragma unroll
            for (int m = 0; m < CP::P; ++m) x[m] = act ? tile[(t + m * CP::T) * NB + k] : make_float2(0.f, 0.f);
            block_fft<LOG_S, CP::LP, +1, false, SyncWarp, CP::SH>(x, xb, t, p.tw_cp, SyncWarp{});
            __syncwarp();
            if (act) {
#pragma unroll
                for (int m = 0; m < CP::P; ++m) {
                    const int j = t + m * CP::T;
                    if (j < gI) tile[j * NB + k] = x[m];
                }
            }
        }
    }
    __syncthreads();
    // ---- inverse real FFT along z of rows j < gI, crop, skip, gate
    const int64_t d = slab % p.D;
    const float dk = p.skip ? __ldg(p.skip + d) : 0.f;
    const int64_t pbase = (slab * gI + i) * (int64_t)gI * gI;
    {
        const int g = tid / R::T, t = tid % R::T;
        float2 *xb = gbuf + g * R::BUF;
        for (int j0 = 0; j0 < gI; j0 += R::G) {
            const int j = j0 + g;
            const bool act = j < gI;
            const float2 *Y = tile + (act ? j : 0) * NB;
            constexpr int PK = gI / 2;
            const int64_t rb = pbase + (int64_t)(act ? j : 0) * gI;
            float2 uu[R::P], gg[R::P];
#pragma unroll
            for (int m = 0; m < R::P; ++m) {
                const int e = t + m * R::T;
                const bool in = act && e < PK;
                uu[m] = (in && dk != 0.f) ? __ldg(reinterpret_cast<const float2 *>(p.u + rb) + e) : make_float2(0.f, 0.f);
                gg[m] = (in && p.gate) ? __ldg(reinterpret_cast<const float2 *>(p.gate + rb) + e) : make_float2(1.f, 1.f);
            }
            float2 x[R::P];
#pragma unroll
            for (int m = 0; m < R::P; ++m) {
                const int k = t + m * R::T;
                float2 yk = Y[k], yn = Y[H2 - k];
                if (k == 0) {                 // DC and Nyquist: real parts only
                    yk.y = 0.f;
                    yn.y = 0.f;
                }
                const float2 A = make_float2(yk.x + yn.x, yk.y - yn.y);      // Y[k] + Y*[H2-k]
                const float2 Bv = make_float2(yk.x - yn.x, yk.y + yn.y);     // Y[k] - Y*[H2-k]
                const float2 cB = cmulc(Bv, wsplit(p.tw_split, k, H2));     // W^-k B
                x[m] = make_float2(A.x - cB.y, A.y + cB.x);                // A + i W^-k B
            }
            block_fft<LOG_S - 1, R::LP, +1, false, SyncWarp, R::SH>(x, xb, t, p.tw_r, SyncWarp{});
            if (act) {
#pragma unroll
                for (int m = 0; m < R::P; ++m) {
                    const int e = t + m * R::T;                 // packed output point
                    if (e < PK) {
                        float2 v = make_float2(x[m].x * p.scale, x[m].y * p.scale);
                        if (dk != 0.f) {
                            v.x = fmaf(dk, uu[m].x, v.x);
                            v.y = fmaf(dk, uu[m].y, v.y);
                        }
                        if (p.gate) {
                            v.x *= gg[m].x;
                            v.y *= gg[m].y;
                        }
                        reinterpret_cast<float2 *>(p.y + rb)[e] = v;
                    }
                }
            }
            __syncwarp();
        }
    }
}

// chunk of slabs whose workspace (gI x S x (S/2+1) complex each) fits ~80 MB
// (80 MB: at the 128^3 transform grid that is 9 spectrum or 18 padded conv
// slabs per chunk, 1152 CTAs per launch = 3.9 waves of two CTAs per SM; the
// 64 MB chunks before gave 3.03 and 3.24 waves and measured 4% slower.)
int64_t nd_chunk(int64_t slabs, int64_t per_slab) {
    int64_t c = ((int64_t)80 << 20) / per_slab;
    if (c < 1) c = 1;
    return c < slabs ? c : slabs;
}

template <typename Kern>
hy_status nd_smem(Kern k, size_t bytes) {
    if (bytes > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
        if (e != cudaSuccess) return set_cuda_error("N-D smem attribute", e);
    }
    return HY_OK;
}

template <int LOG_S>
size_t gbuf_elems() {
    using CP = Grp<LOG_S, nd_col_log_p(LOG_S)>;
    size_t m = (size_t)NT / Grp<LOG_S>::T * Grp<LOG_S>::BUF;
    const size_t r = (size_t)NT / Grp<LOG_S - 1>::T * Grp<LOG_S - 1>::BUF;
    const size_t c = (size_t)NT / CP::T * CP::BUF;
    if (r > m) m = r;
    if (c > m) m = c;
    return m;
}

template <int LOG_S, bool PAD>
hy_status run_nd(const NDArgs &a, NdParams p, cudaStream_t s, bool spec, int64_t slabs, size_t ws_bytes) {
    constexpr int S = 1 << LOG_S;
    constexpr int NB = S / 2 + 1;
    constexpr int gI = PAD ? S / 2 : S;
    p.tw_r = tw_stages(LOG_S - 1, nd_log_p(LOG_S - 1));
    p.tw_c = tw_stages(LOG_S, nd_log_p(LOG_S));
    p.tw_cp = tw_stages(LOG_S, nd_col_log_p(LOG_S));
    p.tw_split = tw_split(LOG_S - 1);
    if (!p.tw_r || !p.tw_c || !p.tw_cp || !p.tw_split) return set_error(HY_ERR_CUDA, "N-D twiddle tables missing");
    const int64_t per_slab = (int64_t)gI * S * NB * 8;
    const int64_t cs = nd_chunk(slabs, per_slab);
    const size_t sm1 = sizeof(float2) * ((size_t)S * NB + gbuf_elems<LOG_S>());
    const size_t sm2 = sizeof(float2) * ((size_t)gI * NB + (size_t)NT / Grp<LOG_S>::T * Grp<LOG_S>::BUF);
    const size_t sm2c = sm2 + sizeof(float2) * 2 * (size_t)S * xpass_hstride<LOG_S>();
    auto k1 = nd_fwd_plane<LOG_S, PAD>;
    auto k2c = nd_xpass<LOG_S, PAD, false>;
    auto k2s = nd_xpass<LOG_S, PAD, true>;
    auto k3 = nd_inv_plane<LOG_S, PAD>;
    hy_status st;
    if ((st = nd_smem(k1, sm1)) != HY_OK || (st = nd_smem(k2c, sm2c)) != HY_OK ||
        (st = nd_smem(k2s, sm2)) != HY_OK || (st = nd_smem(k3, sm1)) != HY_OK)
        return st;
    (void)a;
    // chunks alternate between two streams and two workspace buffers when
    // the workspace holds two (chunk_lanes.h)
    float2 *const ws0 = p.ws;
    LaneScope lanes;
    if ((st = lanes.open(chunk_lanes(slabs, cs, (size_t)per_slab, ws_bytes), s)) != HY_OK) return st;
    int ci = 0;
    for (int64_t s0 = 0; s0 < slabs; s0 += cs, ++ci) {
        const int64_t ns = (slabs - s0) < cs ? (slabs - s0) : cs;
        const cudaStream_t st_ = lanes.stream_of(ci);
        p.ws = ws0 + (int64_t)lanes.lane_of(ci) * cs * (per_slab / 8);
        p.slab0 = s0;
        k1<<<dim3(gI, (unsigned)ns), NT, sm1, st_>>>(p);
        if (spec) {
            k2s<<<dim3(S, (unsigned)ns), NT, sm2, st_>>>(p);
        } else {
            k2c<<<dim3(S, (unsigned)ns), NT, sm2c, st_>>>(p);
            k3<<<dim3(gI, (unsigned)ns), NT, sm1, st_>>>(p);
        }
        if ((st = check_launch("N-D launch")) != HY_OK) return st;
    }
    return lanes.join();
}

bool cube(const int g[3]) { return g[0] == g[1] && g[1] == g[2]; }
int ilog2i(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

}  // namespace

// Workspace: one chunk buffer at least; the queries return one per lane
// that can be busy (chunk_lanes.h).
size_t nd_workspace_of(int64_t slabs, int64_t per, bool minimum) {
    const int64_t cs = nd_chunk(slabs, per);
    return minimum ? (size_t)(cs * per) : chunk_workspace(slabs, cs, (size_t)per);
}

size_t nd_conv_workspace(const int g[3], int circular, int64_t B, int64_t D, bool minimum) {
    if (!cube(g)) return 0;
    const int64_t S = circular ? g[0] : 2 * g[0];
    const int64_t per = (int64_t)g[0] * S * (S / 2 + 1) * 8;
    return nd_workspace_of(B * D, per, minimum);
}

hy_status launch_nd_conv(const NDArgs &a, cudaStream_t s) {
    if (!cube(a.g)) return set_error(HY_ERR_UNSUPPORTED, "hyena_nd_conv: only cubic grids are built");
    NdParams p{};
    p.D = a.D;
    p.u = a.u;
    p.gate = a.gate;
    p.skip = a.skip;
    p.H = a.H;
    p.H_batch_stride = a.H_batch_stride;
    p.ws = reinterpret_cast<float2 *>(a.ws);
    p.y = a.y;
    const int S = a.S[0];
    p.scale = (float)(1.0 / (2.0 * (double)S * S * S));
    const int64_t slabs = a.B * a.D;
    const bool pad = !a.circular;
    switch (ilog2i(S)) {
#define HY_ND(LS) \
    case LS: return pad ? run_nd<LS, true>(a, p, s, false, slabs, a.ws_bytes) : run_nd<LS, false>(a, p, s, false, slabs, a.ws_bytes);
        HY_ND(3) HY_ND(4) HY_ND(5) HY_ND(6) HY_ND(7)
#undef HY_ND
        default: return set_error(HY_ERR_UNSUPPORTED, "hyena_nd_conv: transform edge %d not built", S);
    }
}

size_t nd_spectrum_workspace(int64_t rows, const int S[3], bool minimum) {
    if (!(S[0] == S[1] && S[1] == S[2])) return 0;
    const int64_t per = (int64_t)S[0] * S[0] * (S[0] / 2 + 1) * 8;
    return nd_workspace_of(rows, per, minimum);
}

hy_status launch_nd_spectrum(int64_t rows, const int S[3], const float *h, float2 *H, void *ws, size_t ws_bytes,
                             cudaStream_t s) {
    if (!(S[0] == S[1] && S[1] == S[2]))
        return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: only cubic grids are built");
    NdParams p{};
    p.D = 1;
    p.u = h;
    p.Hout = H;
    p.ws = reinterpret_cast<float2 *>(ws);
    NDArgs a{};
    switch (ilog2i(S[0])) {
#define HY_NS(LS) \
    case LS: return run_nd<LS, false>(a, p, s, true, rows, ws_bytes);
        HY_NS(3) HY_NS(4) HY_NS(5) HY_NS(6) HY_NS(7)
#undef HY_NS
        default: return set_error(HY_ERR_UNSUPPORTED, "hyena_filter_spectrum: transform edge %d not built", S[0]);
    }
}

}  // namespace hy
