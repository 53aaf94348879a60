// filter_gen.cu -- fused implicit filter generator.
//
// [HN] 아키텍처 상세, step 2: h(t) = FFN(pos_enc(t)) · w(t), w(t) = e^{-αt};
// [ES] 어떻게 동작하나요?: a small MLP with sinusoidal features and an
// exponential decay window; [ND] 방법론: HyenaND: coordinate MLP on the N-D
// grid with FiLM conditioning per sample.
//
// One CTA owns P = 64 consecutive positions of one filter set.  It builds
// the positional encoding in shared memory, runs the hidden layers once
// (64-output tiles) and then sweeps the last layer in 128-output tiles;
// only when the grid has fewer CTAs than SMs is the last layer split over
// grid z (each split recomputes the small hidden layers).  Every
// layer is an fp32 GEMM over K = layer input width, accumulated as K outer
// products into a 4-position x CPT-output register tile per thread:
//   activations  act[k][pos]    (one float4 read: 4 positions)
//   weights      wT[k][o]       (transposed while staged; CPT/4 float4 reads)
// so each k costs 1 + CPT/4 shared loads for 4*CPT independent FMAs.  The
// weight tile (with its bias, decay rates and FiLM rows) of the next tile is
// copied with cp.async while the current one is computed (two buffers).
// Hidden outputs get bias, FiLM and the activation and stay in shared
// memory; last-layer outputs get bias and the decay window and go straight
// to HBM as float4 row segments.
#include <cuda_fp16.h>
#include <cstdlib>
#include <cstring>

#include "kernels.h"
#include "status.h"
#include "tcgen05.cuh"

namespace hy {

namespace {

constexpr int P = 64;           // positions per CTA
constexpr int NT = 256;         // threads: 16 position groups x 16 output groups
constexpr int CPT_H = 4;        // outputs per thread, hidden layers (64-output tiles)
constexpr int CPT_L = 8;        // outputs per thread, last layer (128-output tiles)
constexpr int OT_MAX = 16 * CPT_L;
constexpr int OTS = OT_MAX + 4; // wT row stride: = 4 (mod 32) keeps the staging stores conflict-free
constexpr int MAXW = 132;       // max layer input width
constexpr int MAXL = 4;
constexpr int NPAR = 5;         // per-output parameter rows staged with a tile: bias, alpha, gamma, beta, omega

struct GenParams {
    int ndim;
    int64_t L;                  // 1-D length
    int g, S, log_s, circular;  // 3-D
    int F, include_t;
    int nl;
    int widths[MAXL + 1];
    const float *W[MAXL];
    const float *b[MAXL];
    int act;
    const float *gamma, *beta;
    const float *alpha;
    const float *om[MAXL];      // sine frequencies of hidden layer l's units, or NULL
    int window;                 // HY_WIN_EXP / HY_WIN_GAUSS
    int64_t npos;               // positions per set (L or S^3)
    int ka;                     // max layer input width (activation rows)
    int wbuf;                   // floats per weight buffer
    int out_chunk;              // last-layer outputs per grid-z slice (multiple of OT_MAX)
    int vec_out;                // float4 stores of the output rows are aligned
    float *h;
    // resident-weight kernel: float offsets into the resident region
    int r_w[MAXL], r_ws[MAXL];  // wT_l[k][o] at r_w[l] + k * r_ws[l] + o
    int r_b[MAXL], r_om[MAXL];  // biases, sine frequencies (or -1)
    int r_g, r_be, r_al;        // FiLM gamma / beta of the CTA's set (or -1), decay rates
    // tensor-core last layer (resident kernel): operands after the resident region
    int t_kpad;                 // last-layer K rounded up to 16
    int t_katoms;               // 64-element K atoms
    int t_nmt;                  // 128-output M tiles
    uint32_t t_cols;            // TMEM columns (64 per M tile, power of two >= 32)
    uint32_t *fault;            // device fault word
};

constexpr float kLog2e = 1.4426950408889634f;

// x * sigmoid(x); exp(-x) as 2^(-x log2 e) (relative error ~1e-7 |x|)
__device__ __forceinline__ float silu(float a) { return a * __frcp_rn(1.f + exp2f(-a * kLog2e)); }

__device__ __forceinline__ int signed_off(int i, int S) { return i < S / 2 ? i : i - S; }

__device__ __forceinline__ void cpa4(float *smem, const float *g) {
    const unsigned sa = (unsigned)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sa), "l"(g) : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Stage outputs o0 .. o0+rows of layer l: wT[k][r] = W[o0 + r][k] (k < win)
// and the per-output rows par[j][r] (bias; decay rate on the last layer;
// FiLM gamma/beta of this set on the first hidden layer).  A warp copies
// 4 weight rows x 8 consecutive k per instruction: 32-byte global segments,
// and with the row stride = 4 (mod 32) the 32 shared stores hit 32 banks.
// Rows at or past `end` are left as they are (their outputs are not used).
__device__ __forceinline__ void stage_tile(const GenParams &p, int l, int o0, int rows, int end, int set,
                                           float *wT) {
    const int win = p.widths[l];
    const float *W = p.W[l];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rr = lane >> 3, kk = lane & 7;
    for (int r0 = 4 * warp; r0 < rows; r0 += 4 * (NT / 32)) {
        const int r = r0 + rr;
        if (o0 + r >= end) continue;
        const float *src = W + (int64_t)(o0 + r) * win;
        for (int k0 = 0; k0 < win; k0 += 8) {
            const int k = k0 + kk;
            if (k < win) cpa4(wT + k * OTS + r, src + k);
        }
    }
    float *par = wT + p.ka * OTS;
    const bool last = l == p.nl - 1;
    const bool film = l == 0 && !last && p.gamma;
    const int wout = p.widths[l + 1];
    for (int r = threadIdx.x; r < rows; r += NT) {
        const int o = o0 + r;
        if (o >= end) continue;
        cpa4(par + r, p.b[l] + o);
        if (last) cpa4(par + OT_MAX + r, p.alpha + o);
        if (film) {
            cpa4(par + 2 * OT_MAX + r, p.gamma + (int64_t)set * wout + o);
            cpa4(par + 3 * OT_MAX + r, p.beta + (int64_t)set * wout + o);
        }
        if (!last && p.om[l]) cpa4(par + 4 * OT_MAX + r, p.om[l] + o);
    }
}

// acc[a][c] = sum_k act[k][4tx + a] * wT[k][CPT*ty + c], k ascending
// (wT rows ws floats apart).
template <int CPT>
__device__ __forceinline__ void tile_gemm(const float *act, const float *wT, int K, int tx, int ty,
                                          float (&acc)[4][CPT], int ws = OTS) {
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < CPT; ++c) acc[a][c] = 0.f;
    const float *ap = act + 4 * tx;
    const float *wp = wT + CPT * ty;
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        const float4 av = *reinterpret_cast<const float4 *>(ap + k * P);
        const float x[4] = {av.x, av.y, av.z, av.w};
        float w[CPT];
#pragma unroll
        for (int c4 = 0; c4 < CPT / 4; ++c4) {
            const float4 wv = *reinterpret_cast<const float4 *>(wp + k * ws + 4 * c4);
            w[4 * c4 + 0] = wv.x;
            w[4 * c4 + 1] = wv.y;
            w[4 * c4 + 2] = wv.z;
            w[4 * c4 + 3] = wv.w;
        }
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[a][c] = fmaf(w[c], x[a], acc[a][c]);
    }
}

// Positional encoding (a1) of positions p0 .. p0 + P - 1 into act[feature][pos],
// with each position's window argument (t/L or |r|/g) and validity (3-D:
// inside the kernel's support).  scratch (>= 2g floats) is free working space.
__device__ void encode_positions(const GenParams &p, int64_t p0, float *actA, float *scratch, float *s_norm,
                                 int *s_valid) {
    const int tid = threadIdx.x;
    float *actB = scratch;
    const int w0 = p.widths[0];
    if (p.ndim == 1) {
        // integer phase (j t) mod L, then the angle 2 pi r / L; below 2^24
        // every integer involved is exact in float
        const bool narrow = p.L * (int64_t)(p.F + 1) < (1LL << 31) && p.L <= (1 << 24);
        const float Lf = (float)p.L;
        for (int idx = tid; idx < P * w0; idx += NT) {
            const int pos = idx & (P - 1), f = idx / P;
            const int64_t tt = p0 + pos;
            float v = 0.f;
            if (tt < p.npos) {
                if (p.include_t && f == 0) {
                    v = narrow ? __fdiv_rn((float)tt, Lf) : (float)((double)tt / (double)p.L);
                } else {
                    const int ff = f - p.include_t;      // 0..2F-1
                    const int j = (ff < p.F ? ff : ff - p.F) + 1;
                    float arg;
                    if (narrow) {
                        const unsigned r = (unsigned)(j * (int)tt) % (unsigned)p.L;
                        arg = __fdiv_rn((float)(2 * r), Lf);
                    } else {
                        const int64_t r = ((int64_t)j * tt) % p.L;
                        arg = (float)(2.0 * (double)r / (double)p.L);
                    }
                    float sn, cs;
                    sincospif(arg, &sn, &cs);
                    v = (ff < p.F) ? cs : sn;
                }
            }
            actA[f * P + pos] = v;
        }
        for (int pos = tid; pos < P; pos += NT) {
            const int64_t tt = p0 + pos;
            s_valid[pos] = tt < p.npos;
            s_norm[pos] = narrow ? __fdiv_rn((float)tt, Lf) : (float)((double)tt / (double)p.L);
        }
    } else {
        const int S = p.S, ls = p.log_s, twog_m = 2 * p.g - 1;
        const float gf = (float)p.g;
        // every feature is cos or sin of pi m / g for one of the 2g phases m
        // = (j r) mod 2g: tabulate them once (in the second activation buffer,
        // free until the first layer writes it)
        float2 *phase = reinterpret_cast<float2 *>(actB);
        for (int m = tid; m <= twog_m; m += NT) {
            float sn, cs;
            sincospif((float)m / gf, &sn, &cs);
            phase[m] = make_float2(cs, sn);
        }
        __syncthreads();
        for (int idx = tid; idx < P * w0; idx += NT) {
            const int pos = idx & (P - 1), f = idx / P;
            const int64_t q = p0 + pos;
            float v = 0.f;
            if (q < p.npos) {
                const int axis = f / (2 * p.F);
                const int ff = f - axis * 2 * p.F;
                const int j = (ff < p.F ? ff : ff - p.F) + 1;
                const int ia = (int)(q >> (ls * (2 - axis))) & (S - 1);
                const int mm = (j * signed_off(ia, S)) & twog_m;   // (j r) mod 2g, 2g a power of two
                const float2 cs = phase[mm];                       // angle pi j r / g
                v = (ff < p.F) ? cs.x : cs.y;
            }
            actA[f * P + pos] = v;
        }
        for (int pos = tid; pos < P; pos += NT) {
            const int64_t q = p0 + pos;
            int valid = 0;
            float nrm = 0.f;
            if (q < p.npos) {
                const int r0 = signed_off((int)(q >> (2 * ls)) & (S - 1), S);
                const int r1 = signed_off((int)(q >> ls) & (S - 1), S);
                const int r2 = signed_off((int)q & (S - 1), S);
                valid = p.circular || ((abs(r0) < p.g) && (abs(r1) < p.g) && (abs(r2) < p.g));
                nrm = sqrtf((float)(r0 * r0 + r1 * r1 + r2 * r2)) / gf;
            }
            s_valid[pos] = valid;
            s_norm[pos] = nrm;
        }
    }

}

__global__ void __launch_bounds__(NT, 2) filter_gen_kernel(const GenParams p) {
    extern __shared__ __align__(16) float sm[];
    float *actA = sm;                          // [ka][P]
    float *actB = actA + p.ka * P;             // [ka][P]
    float *const wbase = actB + p.ka * P;      // two buffers: wT [ka][OTS], then NPAR x OT_MAX parameters
    __shared__ float s_norm[P];                // decay argument per position (t/L or |r|/g)
    __shared__ int s_valid[P];

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t p0 = (int64_t)blockIdx.x * P;
    const int set = blockIdx.y;
    const int nl = p.nl;
    const int nout = p.widths[nl];
    const int lbeg = blockIdx.z * p.out_chunk;
    const int lend = min(nout, lbeg + p.out_chunk);

    // tile sequence: hidden layers in 64-output tiles, then the last layer's
    // slice in 128-output tiles
    auto tile_rows = [&](int l) { return l == nl - 1 ? 16 * CPT_L : 16 * CPT_H; };
    auto first_o = [&](int l) { return l == nl - 1 ? lbeg : 0; };
    auto end_o = [&](int l) { return l == nl - 1 ? lend : p.widths[l + 1]; };

    int l = 0, o0 = first_o(0);
    stage_tile(p, l, o0, tile_rows(l), end_o(l), set, wbase);
    cpa_commit();

    // ---- positional encoding (a1) into actA[feature][pos]
    encode_positions(p, p0, actA, actB, s_norm, s_valid);

    // ---- MLP layers (a2)
    float *cur = actA, *nxt = actB;
    int buf = 0;
    while (l < nl) {
        // next tile in the sequence, prefetched into the other buffer
        int nl_l = l, nl_o = o0 + tile_rows(l);
        if (nl_o >= end_o(l)) {
            nl_l = l + 1;
            nl_o = nl_l < nl ? first_o(nl_l) : 0;
        }
        if (nl_l < nl) {
            stage_tile(p, nl_l, nl_o, tile_rows(nl_l), end_o(nl_l), set, wbase + (buf ^ 1) * p.wbuf);
            cpa_commit();
            cpa_wait<1>();
        } else {
            cpa_wait<0>();
        }
        __syncthreads();   // weight tile and the previous layer's activations visible

        const float *wT = wbase + buf * p.wbuf;
        const float *par = wT + p.ka * OTS;
        const int K = p.widths[l];
        if (l < nl - 1) {
            float acc[4][CPT_H];
            tile_gemm<CPT_H>(cur, wT, K, tx, ty, acc);
            const int wout = p.widths[l + 1];
            const bool film = (l == 0) && p.gamma;
#pragma unroll
            for (int c = 0; c < CPT_H; ++c) {
                const int r = CPT_H * ty + c;
                const int o = o0 + r;
                if (o >= wout) continue;
                const float bo = par[r];
                const float gm = film ? par[2 * OT_MAX + r] : 0.f;
                const float bt = film ? par[3 * OT_MAX + r] : 0.f;
                const float om = p.om[l] ? par[4 * OT_MAX + r] : 1.f;
                float v[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    float x = acc[a][c] + bo;
                    if (film) x = fmaf(1.f + gm, x, bt);
                    if (p.act == HY_ACT_SILU) x = silu(x);
                    else if (p.act == HY_ACT_SINE) x = sinf(om * x);
                    v[a] = x;
                }
                *reinterpret_cast<float4 *>(nxt + o * P + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
            }
        } else {
            float acc[4][CPT_L];
            tile_gemm<CPT_L>(cur, wT, K, tx, ty, acc);
            float nrm[4];
            bool ok[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                nrm[a] = s_norm[4 * tx + a];
                if (p.window == HY_WIN_GAUSS) nrm[a] *= nrm[a];
                ok[a] = s_valid[4 * tx + a] != 0;
            }
            const int64_t q0 = p0 + 4 * tx;
            const bool full = p.vec_out && q0 + 3 < p.npos;
#pragma unroll
            for (int c = 0; c < CPT_L; ++c) {
                const int r = CPT_L * ty + c;
                const int o = o0 + r;
                if (o >= lend) continue;
                const float bo = par[r];
                const float al = par[OT_MAX + r] * kLog2e;      // e^{-a n} = 2^{-a log2(e) n}
                float v[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) v[a] = ok[a] ? (acc[a][c] + bo) * exp2f(-al * nrm[a]) : 0.f;   // nrm: n or n^2
                float *dst = p.h + ((int64_t)set * nout + o) * p.npos + q0;
                if (full) {
                    *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
                } else {
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        if (q0 + a < p.npos) dst[a] = v[a];
                }
            }
        }
        __syncthreads();   // all reads of this weight buffer and of cur done
        if (nl_l != l) {
            float *t = cur;
            cur = nxt;
            nxt = t;
        }
        l = nl_l;
        o0 = nl_o;
        buf ^= 1;
    }
}

// ---- tensor-core last layer: fp16 hi/lo operands in the K-major
// 128-byte-swizzled layout (64 K elements per 128-byte row, 8-row atoms)
constexpr int TC_A_ATOM = 128 * 128;   // bytes of one K atom of a 128-row A tile
constexpr int TC_B_ATOM = P * 128;     // bytes of one K atom of the 64-row B tile

__device__ __forceinline__ uint32_t fg_sw128(int r, int k) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((((k & 63) >> 3) ^ (r & 7)) << 4) + (k & 7) * 2);
}
__device__ __forceinline__ void fp16_split(float x, __half &hi, __half &lo) {
    hi = __float2half_rn(x);
    lo = __float2half_rn(x - __half2float(hi));
}

// ----------------------------------------------------------------------------
// Resident-weight variant, for many position tiles per filter set: every
// layer's weights (transposed: wT_l[k][o]) and per-output parameters (bias,
// sine frequencies, this set's FiLM rows, decay rates) are loaded into
// shared memory once; the CTA then walks position tiles blockIdx.x,
// blockIdx.x + gridDim.x, ... of set blockIdx.y.  The arithmetic per tile is
// the streaming kernel's (same tile GEMMs, same epilogues).
// ----------------------------------------------------------------------------
template <bool TC>
__global__ void __launch_bounds__(NT, 2) filter_gen_resident_kernel(const GenParams p, int64_t res_floats) {
    extern __shared__ __align__(16) float sm[];
    float *actA = sm;                          // [ka][P]
    float *actB = actA + p.ka * P;             // [ka][P]
    float *res = actB + p.ka * P;              // resident weights and parameters
    __shared__ float s_norm[P];
    __shared__ int s_valid[P];
    // tensor-core operands (1024-byte aligned): A hi, A lo (last-layer W), B hi, B lo (its inputs)
    uint8_t *tcb = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(res + res_floats) + 1023) & ~uintptr_t(1023));
    const int a_part = p.t_nmt * p.t_katoms * TC_A_ATOM, b_part = p.t_katoms * TC_B_ATOM;
    uint8_t *a_hi = tcb, *a_lo = tcb + a_part, *b_hi = tcb + 2 * a_part, *b_lo = b_hi + b_part;
    __shared__ uint32_t s_tmem;
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int set = blockIdx.y;
    const int nl = p.nl;
    const int nout = p.widths[nl];
    const int64_t nblk = (p.npos + P - 1) / P;

    if (TC) {
        if ((tid >> 5) == 0) tc::tmem_alloc(&s_tmem, p.t_cols);
        if (tid == 0) {
            mbar_init(&s_bar, 1);
            mbar_init_fence();
            s_abort = 0;
        }
        // A: last-layer weights, rows = outputs (zero past nout), K = inputs (zero past K)
        const int K = p.widths[nl - 1];
        const float *W = p.W[nl - 1];
        const int rows = p.t_nmt * 128;
        for (int idx = tid; idx < rows * p.t_kpad; idx += NT) {
            const int o = idx / p.t_kpad, k = idx - o * p.t_kpad;
            const float v = (o < nout && k < K) ? __ldg(W + (int64_t)o * K + k) : 0.f;
            __half hi, lo;
            fp16_split(v, hi, lo);
            const uint32_t off = (uint32_t)((o >> 7) * p.t_katoms * TC_A_ATOM + (k >> 6) * TC_A_ATOM) + fg_sw128(o & 127, k);
            *reinterpret_cast<__half *>(a_hi + off) = hi;
            *reinterpret_cast<__half *>(a_lo + off) = lo;
        }
        // B: the K padding stays zero (the hidden epilogue writes k < K only)
        for (int idx = tid; idx < 2 * b_part / 16; idx += NT) reinterpret_cast<uint4 *>(b_hi)[idx] = make_uint4(0, 0, 0, 0);
    }
    for (int l = 0; l < nl; ++l) {
        const int win = p.widths[l], wout = p.widths[l + 1];
        const float *W = p.W[l];
        float *wT = res + p.r_w[l];
        if (!(TC && l == nl - 1))
            for (int idx = tid; idx < win * wout; idx += NT) {    // W row-major (out x in): reads along k
                const int o = idx / win, k = idx - o * win;
                wT[k * p.r_ws[l] + o] = __ldg(W + idx);
            }
        for (int o = tid; o < wout; o += NT) {
            res[p.r_b[l] + o] = __ldg(p.b[l] + o);
            if (p.r_om[l] >= 0) res[p.r_om[l] + o] = __ldg(p.om[l] + o);
            if (l == 0 && p.r_g >= 0) {
                res[p.r_g + o] = __ldg(p.gamma + (int64_t)set * wout + o);
                res[p.r_be + o] = __ldg(p.beta + (int64_t)set * wout + o);
            }
        }
    }
    for (int o = tid; o < nout; o += NT) res[p.r_al + o] = __ldg(p.alpha + o) * kLog2e;   // e^{-a n} = 2^{-a log2(e) n}

    if (TC) {
        fence_proxy_async_smem();              // the A operand is read by the tensor cores
        tc::fence_before();
    }
    uint32_t tc_phase = 0;
    for (int64_t bt = blockIdx.x; bt < nblk; bt += gridDim.x) {
        const int64_t p0 = bt * P;
        __syncthreads();                       // resident region written / previous tile's reads done
        if (TC) {
            tc::fence_after();
            if (s_abort) break;                // uniform: read between two barriers
        }
        encode_positions(p, p0, actA, actB, s_norm, s_valid);
        __syncthreads();
        float *cur = actA, *nxt = actB;
        for (int l = 0; l < nl; ++l) {
            const int K = p.widths[l];
            const float *wT = res + p.r_w[l];
            if (l < nl - 1) {
                const int wout = p.widths[l + 1];
                const bool film = (l == 0) && p.r_g >= 0;
                for (int o0 = 0; o0 < wout; o0 += 16 * CPT_H) {
                    float acc[4][CPT_H];
                    tile_gemm<CPT_H>(cur, wT + o0, K, tx, ty, acc, p.r_ws[l]);
#pragma unroll
                    for (int c = 0; c < CPT_H; ++c) {
                        const int o = o0 + CPT_H * ty + c;
                        if (o >= wout) continue;
                        const float bo = res[p.r_b[l] + o];
                        const float gm = film ? res[p.r_g + o] : 0.f;
                        const float bt2 = film ? res[p.r_be + o] : 0.f;
                        const float om = p.r_om[l] >= 0 ? res[p.r_om[l] + o] : 1.f;
                        float v[4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) {
                            float x = acc[a][c] + bo;
                            if (film) x = fmaf(1.f + gm, x, bt2);
                            if (p.act == HY_ACT_SILU) x = silu(x);
                            else if (p.act == HY_ACT_SINE) x = sinf(om * x);
                            v[a] = x;
                        }
                        if (TC && l == nl - 2) {
                            // inputs of the tensor-core last layer: B[pos][k = o], fp16 hi and lo
#pragma unroll
                            for (int a = 0; a < 4; ++a) {
                                __half hi, lo;
                                fp16_split(v[a], hi, lo);
                                const int pos = 4 * tx + a;
                                const uint32_t off = (uint32_t)((o >> 6) * TC_B_ATOM) + fg_sw128(pos, o);
                                *reinterpret_cast<__half *>(b_hi + off) = hi;
                                *reinterpret_cast<__half *>(b_lo + off) = lo;
                            }
                        } else {
                            *reinterpret_cast<float4 *>(nxt + o * P + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
                        }
                    }
                }
                if (TC && l == nl - 2) fence_proxy_async_smem();   // the B operand is read by the tensor cores
                __syncthreads();
                float *t2 = cur;
                cur = nxt;
                nxt = t2;
            } else if (TC) {
                // D[o][pos] = Σ_k W[o][k] act[pos][k] on the tensor cores: hi·hi + hi·lo + lo·hi
                if (tid == 0) {
                    tc::fence_after();
                    constexpr uint32_t IDESC = tc::idesc_f16(128, P, false);
                    for (int mt = 0; mt < p.t_nmt; ++mt) {
                        bool first = true;
                        for (int term = 0; term < 3; ++term) {
                            const uint8_t *A = (term == 2 ? a_lo : a_hi) + mt * p.t_katoms * TC_A_ATOM;
                            const uint8_t *Bm = term == 1 ? b_lo : b_hi;
                            for (int ks = 0; ks < p.t_kpad / 16; ++ks) {
                                const uint64_t ad = tc::desc_k_sw128(smem_u32(A + (ks >> 2) * TC_A_ATOM)) + 2 * (ks & 3);
                                const uint64_t bd = tc::desc_k_sw128(smem_u32(Bm + (ks >> 2) * TC_B_ATOM)) + 2 * (ks & 3);
                                tc::mma_f16(s_tmem + 64u * mt, ad, bd, IDESC, first ? 0u : 1u);
                                first = false;
                            }
                        }
                    }
                    tc::commit(&s_bar);
                    if (!mbar_wait_sleep(&s_bar, tc_phase)) {
                        record_fault(p.fault, HY_FAULT_FILTER_MMA);
                        s_abort = 1;
                    }
                }
                tc_phase ^= 1;
                __syncthreads();
                tc::fence_after();
                // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (outputs) and
                // positions 32 (w / 4) .. + 31 of each M tile
                const int warp = tid >> 5, lane = tid & 31;
                const int q = warp & 3, hc = warp >> 2;
                for (int mt = 0; mt < p.t_nmt; ++mt) {
                    __syncwarp();                      // tcgen05.ld is warp-wide
                    uint32_t v[32];
                    tc::tmem_ld32(s_tmem + ((uint32_t)(32 * q) << 16) + 64u * mt + 32u * hc, v);
                    tc::tmem_wait_ld();
                    const int o = 128 * mt + 32 * q + lane;
                    if (o >= nout) continue;
                    const float bo = res[p.r_b[l] + o];
                    const float al = res[p.r_al + o];
                    const int64_t q0 = p0 + 32 * hc;
                    float *dst = p.h + ((int64_t)set * nout + o) * p.npos + q0;
                    float w[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        float nr = s_norm[32 * hc + j];
                        if (p.window == HY_WIN_GAUSS) nr *= nr;
                        w[j] = s_valid[32 * hc + j] ? (__uint_as_float(v[j]) + bo) * exp2f(-al * nr) : 0.f;
                    }
                    if (p.vec_out && q0 + 31 < p.npos) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(dst + j) = make_float4(w[j], w[j + 1], w[j + 2], w[j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (q0 + j < p.npos) dst[j] = w[j];
                    }
                }
                tc::fence_before();
            } else {
                float nrm[4];
                bool ok[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    nrm[a] = s_norm[4 * tx + a];
                    if (p.window == HY_WIN_GAUSS) nrm[a] *= nrm[a];
                    ok[a] = s_valid[4 * tx + a] != 0;
                }
                const int64_t q0 = p0 + 4 * tx;
                const bool full = p.vec_out && q0 + 3 < p.npos;
                for (int o0 = 0; o0 < nout; o0 += 16 * CPT_L) {
                    float acc[4][CPT_L];
                    tile_gemm<CPT_L>(cur, wT + o0, K, tx, ty, acc, p.r_ws[l]);
#pragma unroll
                    for (int c = 0; c < CPT_L; ++c) {
                        const int o = o0 + CPT_L * ty + c;
                        if (o >= nout) continue;
                        const float bo = res[p.r_b[l] + o];
                        const float al = res[p.r_al + o];
                        float v[4];
#pragma unroll
                        for (int a = 0; a < 4; ++a) v[a] = ok[a] ? (acc[a][c] + bo) * exp2f(-al * nrm[a]) : 0.f;
                        float *dst = p.h + ((int64_t)set * nout + o) * p.npos + q0;
                        if (full) {
                            *reinterpret_cast<float4 *>(dst) = make_float4(v[0], v[1], v[2], v[3]);
                        } else {
#pragma unroll
                            for (int a = 0; a < 4; ++a)
                                if (q0 + a < p.npos) dst[a] = v[a];
                        }
                    }
                }
            }
        }
    }
    if (TC) {
        // no MMA may still be running when TMEM is freed (all were waited on;
        // this covers one whose wait gave up)
        if (tid == 0) {
            tc::commit(&s_bar);
            if (!mbar_wait_sleep(&s_bar, tc_phase)) record_fault(p.fault, HY_FAULT_FILTER_MMA);
        }
        tc::fence_before();
        __syncthreads();
        tc::fence_after();
        __syncwarp();
        if ((tid >> 5) == 0) tc::tmem_free(s_tmem, p.t_cols);
    }
}

// The tensor-core last layer is opt-in (HYENA_FILTER_ENGINE=tensor).
bool tensor_last_layer_enabled() {
    const char *e = std::getenv("HYENA_FILTER_ENGINE");
    return e && std::strcmp(e, "tensor") == 0;
}

// Float layout of the resident region; returns its size in floats.  Each
// weight matrix is padded by one tile of columns so the tile GEMMs of the
// last (partial) output tile stay inside the region.
int64_t resident_layout(GenParams &p, bool last_on_tensor_cores) {
    int64_t off = 0;
    auto take = [&](int64_t n) { const int64_t o = off; off += (n + 3) & ~int64_t(3); return (int)o; };
    for (int l = 0; l < p.nl; ++l) {
        const int wout = p.widths[l + 1];
        p.r_ws[l] = (wout + 3) & ~3;
        const bool skip = last_on_tensor_cores && l == p.nl - 1;   // held as the MMA operand instead
        p.r_w[l] = take(skip ? 0 : (int64_t)p.widths[l] * p.r_ws[l] + 16 * CPT_L);
        p.r_b[l] = take(wout);
        p.r_om[l] = p.om[l] ? take(wout) : -1;
    }
    const bool film = p.gamma && p.nl > 1;
    p.r_g = film ? take(p.widths[1]) : -1;
    p.r_be = film ? take(p.widths[1]) : -1;
    p.r_al = take(p.widths[p.nl]);
    return off;
}

}  // namespace

hy_status launch_filter_gen(const hy_filter_desc &d, float *h, cudaStream_t s) {
    GenParams p{};
    p.ndim = d.ndim;
    p.L = d.L;
    p.g = d.grid;
    p.circular = d.circular;
    p.S = d.circular ? d.grid : 2 * d.grid;
    p.log_s = 0;
    while ((1 << p.log_s) < p.S) ++p.log_s;
    p.F = d.n_freq;
    p.include_t = d.include_t;
    p.nl = d.n_layers;
    if (p.nl < 1 || p.nl > MAXL) return set_error(HY_ERR_UNSUPPORTED, "n_layers must be 1..%d", MAXL);
    p.ka = 1;
    for (int l = 0; l <= p.nl; ++l) {
        p.widths[l] = d.widths[l];
        if (l < p.nl) {
            if (d.widths[l] > MAXW) return set_error(HY_ERR_UNSUPPORTED, "layer input width %d > %d", d.widths[l], MAXW);
            p.ka = d.widths[l] > p.ka ? d.widths[l] : p.ka;
        }
    }
    for (int l = 0; l < p.nl; ++l) {
        p.W[l] = d.W[l];
        p.b[l] = d.b[l];
    }
    p.act = d.act;
    for (int l = 0, off = 0; l < p.nl; ++l) {
        p.om[l] = (d.act == HY_ACT_SINE && d.omega && l < p.nl - 1) ? d.omega + off : nullptr;
        if (l < p.nl - 1) off += d.widths[l + 1];
    }
    p.window = d.window;
    p.gamma = d.film_gamma;
    p.beta = d.film_beta;
    p.alpha = d.alpha;
    p.npos = d.ndim == 1 ? (int64_t)d.L : (int64_t)p.S * p.S * p.S;
    p.vec_out = (p.npos % 4 == 0) && ((uintptr_t)h % 16 == 0);
    p.h = h;
    p.wbuf = p.ka * OTS + NPAR * OT_MAX;       // a multiple of 4 floats: buffers stay 16-byte aligned
    const int64_t nblk = (p.npos + P - 1) / P;
    if (nblk > 0x7fffffffLL || d.n_sets > 65535) return set_error(HY_ERR_UNSUPPORTED, "filter grid too large");
    int sms = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    // Many position tiles per set, weights that fit in shared memory: keep
    // them resident in persistent CTAs instead of staging them per tile; the
    // last layer runs on the tensor cores when it has a hidden layer before it
    // and K <= 128 (its operands follow the resident region).
    {
        GenParams q = p;
        const int Klast = q.widths[q.nl - 1];
        const int nlast = q.widths[q.nl];
        // (the tensor-core last layer is built and tested but slower than the
        // FP32 pipes here: its fp16 operand stores conflict in shared memory)
        const bool tc = tensor_last_layer_enabled() && q.nl >= 2 && Klast <= 128 && nlast <= 512;
        const int64_t rfl = resident_layout(q, tc);
        size_t tc_bytes = 0;
        if (tc) {
            q.t_kpad = (Klast + 15) & ~15;
            q.t_katoms = (q.t_kpad + 63) / 64;
            q.t_nmt = (nlast + 127) / 128;
            q.t_cols = q.t_nmt <= 1 ? 64u : (q.t_nmt <= 2 ? 128u : 256u);
            q.fault = device_fault_word();
            if (!q.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
            tc_bytes = 1024 + (size_t)2 * q.t_nmt * q.t_katoms * TC_A_ATOM + (size_t)2 * q.t_katoms * TC_B_ATOM;
        }
        const size_t rsmem = sizeof(float) * ((size_t)2 * q.ka * P + (size_t)rfl) + tc_bytes;
        // FP32-pipe last layer: only with two CTAs per SM (with one, the FP32
        // pipes idle at every barrier and the streaming kernel's two CTAs per
        // SM are faster).  Tensor-core last layer: one CTA per SM is enough.
        const bool two = rsmem <= (size_t)113 * 1024;
        if (nblk * d.n_sets >= (int64_t)8 * sms && (two || (tc && rsmem <= (size_t)227 * 1024))) {
            auto kernel = tc ? filter_gen_resident_kernel<true> : filter_gen_resident_kernel<false>;
            cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem);
            if (e != cudaSuccess) return set_cuda_error("filter_gen resident smem attribute", e);
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return set_cuda_error("filter_gen carve-out attribute", e);
            // two CTAs per SM when they fit (TMEM <= 256 columns each), else one
            int64_t per_set = ((int64_t)(two ? 2 : 1) * sms + d.n_sets - 1) / d.n_sets;
            if (per_set > nblk) per_set = nblk;
            dim3 grid((unsigned)per_set, (unsigned)d.n_sets, 1);
            kernel<<<grid, NT, rsmem, s>>>(q, rfl);
            return check_launch("filter_gen (resident weights) launch");
        }
    }
    const size_t smem = sizeof(float) * ((size_t)2 * p.ka * P + (size_t)2 * p.wbuf);
    cudaError_t e = cudaFuncSetAttribute(filter_gen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return set_cuda_error("filter_gen smem attribute", e);
    // split the last layer over grid z only when there are fewer CTAs than
    // SMs (each split recomputes the hidden layers)
    const int nout = d.widths[d.n_layers];
    const int64_t base = nblk * d.n_sets;
    const int ntile = (nout + OT_MAX - 1) / OT_MAX;
    int chunks = 1;
    if (base < (int64_t)sms) chunks = (int)((sms + base - 1) / base);
    if (chunks > ntile) chunks = ntile;
    const int per = (ntile + chunks - 1) / chunks;
    p.out_chunk = per * OT_MAX;
    chunks = (ntile + per - 1) / per;
    dim3 grid((unsigned)nblk, (unsigned)d.n_sets, (unsigned)chunks);
    filter_gen_kernel<<<grid, NT, smem, s>>>(p);
    return check_launch("filter_gen launch");
}

}  // namespace hy
