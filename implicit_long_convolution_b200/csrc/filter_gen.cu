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
// to HBM as float4 row segments.  With many positions per filter set the
// weights stay resident in persistent CTAs, and the layers run on the
// tensor cores where their shapes allow: every layer of a one-hidden-layer
// MLP (filter_gen_tc2_kernel), every layer of a two-hidden-layer MLP over
// few positions with many outputs (filter_gen_tc3_kernel), else the last
// layer (filter_gen_tc_kernel).
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
    // tensor-core last layer: operands after the resident region
    int t_kpad;                 // last-layer K rounded up to 16
    int t_katoms;               // 64-element K atoms
    int t_npad;                 // outputs of a CTA's slice rounded up to 16 (MMA N, in chunks of <= 256)
    int t_slice;                // outputs per grid-z slice (all of them, or 256 when split)
    int t_hpad;                 // hidden units rounded up to 16 (both layers on the tensor cores)
    int t_h2pad;                // second hidden layer's units rounded up to 16 (three layers)
    int t_nslices;              // output slices of t_slice outputs (three layers)
    uint32_t t_cols;            // TMEM columns (power of two >= max(32, t_npad))
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

// ----------------------------------------------------------------------------
// Resident-weight variant, for many position tiles per filter set: every
// layer's weights (transposed: wT_l[k][o]) and per-output parameters (bias,
// sine frequencies, this set's FiLM rows, decay rates) are loaded into
// shared memory once; the CTA then walks position tiles blockIdx.x,
// blockIdx.x + gridDim.x, ... of set blockIdx.y.  The arithmetic per tile is
// the streaming kernel's (same tile GEMMs, same epilogues).
// ----------------------------------------------------------------------------

// Loads the resident region (hidden layers and, unless `skip_last`, the last
// layer's transposed weights; every layer's bias and sine frequencies; the
// set's FiLM rows; the decay rates times log2 e).
__device__ void load_resident(const GenParams &p, float *res, int set, bool skip_last) {
    const int tid = threadIdx.x;
    const int nl = p.nl;
    for (int l = 0; l < nl; ++l) {
        const int win = p.widths[l], wout = p.widths[l + 1];
        const float *W = p.W[l];
        float *wT = res + p.r_w[l];
        if (!(skip_last && l == nl - 1))
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
    for (int o = tid; o < p.widths[nl]; o += NT) res[p.r_al + o] = __ldg(p.alpha + o) * kLog2e;   // e^{-a n} = 2^{-a log2(e) n}
}

// Positional encoding and hidden layers of the P positions from p0 with the
// resident weights; returns the buffer holding the last hidden layer's
// outputs ([width][P]; the encoding itself when there is no hidden layer).
// Ends with a CTA barrier.
__device__ float *resident_hidden(const GenParams &p, const float *res, int64_t p0, float *actA, float *actB,
                                  float *s_norm, int *s_valid) {
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    encode_positions(p, p0, actA, actB, s_norm, s_valid);
    __syncthreads();
    float *cur = actA, *nxt = actB;
    for (int l = 0; l < p.nl - 1; ++l) {
        const int K = p.widths[l];
        const float *wT = res + p.r_w[l];
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
                *reinterpret_cast<float4 *>(nxt + o * P + 4 * tx) = make_float4(v[0], v[1], v[2], v[3]);
            }
        }
        __syncthreads();
        float *t2 = cur;
        cur = nxt;
        nxt = t2;
    }
    return cur;
}

__global__ void __launch_bounds__(NT, 2) filter_gen_resident_kernel(const GenParams p) {
    extern __shared__ __align__(16) float sm[];
    float *actA = sm;                          // [ka][P]
    float *actB = actA + p.ka * P;             // [ka][P]
    float *res = actB + p.ka * P;              // resident weights and parameters
    __shared__ float s_norm[P];
    __shared__ int s_valid[P];

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int set = blockIdx.y;
    const int nl = p.nl;
    const int nout = p.widths[nl];
    const int64_t nblk = (p.npos + P - 1) / P;
    load_resident(p, res, set, false);
    const int l = nl - 1;
    const int K = p.widths[l];
    const float *wT = res + p.r_w[l];
    for (int64_t bt = blockIdx.x; bt < nblk; bt += gridDim.x) {
        const int64_t p0 = bt * P;
        __syncthreads();                       // resident region written / previous tile's reads done
        const float *cur = resident_hidden(p, res, p0, actA, actB, s_norm, s_valid);
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

// ----------------------------------------------------------------------------
// Tensor-core last layer (the dense contraction: 85-97% of the MACs).  A tile
// is TP = 128 positions of one set, the M of one tcgen05 MMA:
//   D[pos][o] = sum_k act[pos][k] W[o][k]
// with both operands K-major in the 128-byte-swizzled layout: A = the last
// hidden layer's outputs of the tile (rows = positions), B = the last layer's
// weights (rows = outputs), held for the whole kernel.  Each operand is split
// into fp16 hi + lo (|x - hi - lo| <= 2^-22 |x|) and the three products
// hi.hi + hi.lo + lo.hi accumulate in fp32 in tensor memory: 128 lanes (the
// positions) x the padded outputs.  The hidden layers run on the FP32 pipes
// (resident weights, two halves of 64 positions); their fp32 outputs are
// packed into A as 16-byte chunks (one position row per thread, swizzled, so
// the stores do not conflict).  The epilogue reads a row per thread from
// tensor memory -- all outputs of one position -- adds the bias, applies the
// decay window and stores: at each output the 32 lanes of a warp write 32
// consecutive positions, one 128-byte segment.  One thread issues the MMAs
// and waits for them (bounded, HY_FAULT_FILTER_MMA).
// ----------------------------------------------------------------------------
constexpr int TP = 2 * P;                 // positions per tensor-core tile
constexpr int TC_ROW = 128;               // bytes per operand row and K atom (64 fp16)

// Byte offset of 16-byte chunk c (k = 8c .. 8c+7 within the atom) of row r in
// a K-major 128-byte-swizzled atom column (8-row groups 1024 bytes apart).
__device__ __forceinline__ uint32_t sw128_chunk(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}
__device__ __forceinline__ void split_h2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}

__global__ void __launch_bounds__(NT, 2) filter_gen_tc_kernel(const GenParams p, int64_t res_floats) {
    extern __shared__ __align__(16) float sm[];
    float *actA = sm;                          // [ka][P]
    float *actB = actA + p.ka * P;             // [ka][P]
    float *res = actB + p.ka * P;              // resident hidden weights and parameters
    // operands (1024-byte aligned): A hi, A lo ([katoms][TP rows][128 B]), B hi, B lo ([katoms][npad rows][128 B])
    uint8_t *tcb = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(res + res_floats) + 1023) & ~uintptr_t(1023));
    const int katoms = p.t_katoms, npad = p.t_npad;
    const int a_part = katoms * TP * TC_ROW, b_part = katoms * npad * TC_ROW;
    uint8_t *a_hi = tcb, *a_lo = tcb + a_part, *b_hi = tcb + 2 * a_part, *b_lo = b_hi + b_part;
    __shared__ float s_norm[TP];
    __shared__ int s_valid[TP];
    __shared__ uint32_t s_tmem;
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int set = blockIdx.y;
    const int nl = p.nl;
    const int nout = p.widths[nl];
    const int obase = blockIdx.z * p.t_slice;  // this CTA's outputs: obase .. obase + t_slice - 1
    const int oend = min(nout, obase + p.t_slice);
    const int K = p.widths[nl - 1];
    const int kchunks = p.t_kpad / 8;          // 16-byte chunks of a row
    const int64_t ntiles = (p.npos + TP - 1) / TP;

    if (warp == 0) tc::tmem_alloc(&s_tmem, p.t_cols);
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    load_resident(p, res, set, true);
    // B: the last layer's weights of the slice, rows obase + o for o < npad
    // (zero past the slice), K padded with zeros
    {
        const float *W = p.W[nl - 1];
        for (int idx = tid; idx < npad * kchunks; idx += NT) {
            const int o = idx / kchunks, c = idx - o * kchunks;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = 8 * c + j;
                v[j] = (obase + o < oend && k < K) ? __ldg(W + (int64_t)(obase + o) * K + k) : 0.f;
            }
            uint4 hi, lo;
            split_h2(v[0], v[1], hi.x, lo.x);
            split_h2(v[2], v[3], hi.y, lo.y);
            split_h2(v[4], v[5], hi.z, lo.z);
            split_h2(v[6], v[7], hi.w, lo.w);
            const uint32_t off = (uint32_t)((c >> 3) * npad * TC_ROW) + sw128_chunk(o, c & 7);
            *reinterpret_cast<uint4 *>(b_hi + off) = hi;
            *reinterpret_cast<uint4 *>(b_lo + off) = lo;
        }
    }
    fence_proxy_async_smem();                  // B is read by the tensor cores
    tc::fence_before();
    uint32_t phase = 0;
    for (int64_t bt = blockIdx.x; bt < ntiles; bt += gridDim.x) {
        __syncthreads();                       // operands / TMEM of the previous tile released
        tc::fence_after();
        if (s_abort) break;                    // uniform: read between two barriers
        // ---- hidden layers of the two halves, packed into A
        for (int half = 0; half < 2; ++half) {
            const int64_t p0 = bt * TP + half * P;
            const float *cur = resident_hidden(p, res, p0, actA, actB, s_norm + half * P, s_valid + half * P);
            for (int idx = tid; idx < P * kchunks; idx += NT) {
                const int r = idx & (P - 1), c = idx / P;
                float v[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int k = 8 * c + j;
                    v[j] = k < K ? cur[k * P + r] : 0.f;
                }
                uint4 hi, lo;
                split_h2(v[0], v[1], hi.x, lo.x);
                split_h2(v[2], v[3], hi.y, lo.y);
                split_h2(v[4], v[5], hi.z, lo.z);
                split_h2(v[6], v[7], hi.w, lo.w);
                const int row = half * P + r;
                const uint32_t off = (uint32_t)((c >> 3) * TP * TC_ROW) + sw128_chunk(row, c & 7);
                *reinterpret_cast<uint4 *>(a_hi + off) = hi;
                *reinterpret_cast<uint4 *>(a_lo + off) = lo;
            }
            __syncthreads();                   // cur is overwritten by the next half
        }
        fence_proxy_async_smem();              // A is read by the tensor cores
        __syncthreads();
        // ---- D = A B^T in up to two N chunks of <= 256 outputs: hi.hi + hi.lo + lo.hi
        if (tid == 0) {
            tc::fence_after();
            for (int n0 = 0; n0 < npad; n0 += 256) {
                const int nc = npad - n0 < 256 ? npad - n0 : 256;
                const uint32_t idesc = tc::idesc_f16(128, nc, false);
                bool first = true;
                for (int term = 0; term < 3; ++term) {
                    const uint8_t *A = term == 2 ? a_lo : a_hi;
                    const uint8_t *Bm = (term == 1 ? b_lo : b_hi) + n0 * TC_ROW;
                    for (int ks = 0; ks < p.t_kpad / 16; ++ks) {
                        const uint64_t ad = tc::desc_k_sw128(smem_u32(A + (ks >> 2) * TP * TC_ROW)) + 2 * (ks & 3);
                        const uint64_t bd = tc::desc_k_sw128(smem_u32(Bm + (ks >> 2) * npad * TC_ROW)) + 2 * (ks & 3);
                        tc::mma_f16(s_tmem + (uint32_t)n0, ad, bd, idesc, first ? 0u : 1u);
                        first = false;
                    }
                }
            }
            tc::commit(&s_bar);
            if (!mbar_wait_sleep(&s_bar, phase)) {
                record_fault(p.fault, HY_FAULT_FILTER_MMA);
                s_abort = 1;
            }
        }
        phase ^= 1;
        __syncthreads();
        tc::fence_after();
        // ---- epilogue: warp w takes positions 32 (w % 4) + lane (TMEM lanes)
        //      and every other 16-column chunk from w / 4
        {
            const int q = warp & 3;
            const int pos = 32 * q + lane;
            const int64_t qq = bt * TP + pos;
            float nr = s_norm[pos];
            if (p.window == HY_WIN_GAUSS) nr *= nr;
            const bool ok = s_valid[pos] != 0;
            const bool in = qq < p.npos;
            const float *bias = res + p.r_b[nl - 1];
            const float *al = res + p.r_al;
            const float nrn = ok ? -nr : 0.f;
            for (int c0 = 16 * (warp >> 2); c0 < npad; c0 += 32) {
                __syncwarp();                  // tcgen05.ld is warp-wide
                uint32_t v[16];
                tc::tmem_ld16(s_tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)c0, v);
                tc::tmem_wait_ld();
                const int ob = obase + c0;
                float *dst = p.h + ((int64_t)set * nout + ob) * p.npos + qq;
#pragma unroll
                for (int j = 0; j < 16; ++j, dst += p.npos) {
                    if (ob + j < oend && in) {
                        const float y = (__uint_as_float(v[j]) + bias[ob + j]) * exp2f(al[ob + j] * nrn);
                        *dst = ok ? y : 0.f;
                    }
                }
            }
        }
        tc::fence_before();
    }
    // no MMA may still be running when TMEM is freed (all were waited on;
    // this covers one whose wait gave up)
    if (tid == 0) {
        tc::commit(&s_bar);
        if (!mbar_wait_sleep(&s_bar, phase)) record_fault(p.fault, HY_FAULT_FILTER_MMA);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    __syncwarp();
    if (warp == 0) tc::tmem_free(s_tmem, p.t_cols);
}

// ----------------------------------------------------------------------------
// Both layers on the tensor cores, for MLPs with one hidden layer (input
// width <= 63, hidden width <= 64).  A tile is 128 positions of one set (the
// MMA M; warps w and w + 4 share TMEM lanes 32 (w % 4) .. + 31, one position
// per thread).  Each thread writes its position's encoding straight into the
// first operand row (fp16 hi/lo, K-major, 128-byte swizzle), with the columns
// permuted so that the cos and sin of one frequency sit side by side (one
// phase gives both) and a constant-1 column after them.  The first-layer
// weights are held with the set's FiLM scale (1 + gamma), the sine
// frequencies and the bias folded in (the bias as the weight of the constant
// column), so the first MMA leaves the activation's argument itself in
// tensor memory.  Each thread reads half of its row back, applies the
// activation and writes the second operand row over the first; the second
// MMA gives the outputs of the CTA's slice (the output bias folded in the
// same way when the hidden width leaves a free column), and the epilogue
// adds the decay window and stores as filter_gen_tc_kernel's does.
// ----------------------------------------------------------------------------
constexpr uint32_t TC2_OUT_COL = 128;     // TMEM column of the output accumulator

// PTX approximate 2^x and 1/x (one MUFU operation each; subnormal results flush to zero)
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_fast(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Encoding feature (its index in the positional encoding's own order) held
// in operand column k: pairs (cos, sin) of each frequency first, then t/L
// (1-D with include_t); -1 for the constant-1 column, -2 for a zero column.
__device__ __forceinline__ int tc2_feature_of_column(const GenParams &p, int k, int npairs) {
    if (k < 2 * npairs) {
        const int pp = k >> 1, s = k & 1;
        if (p.ndim == 1) return p.include_t + s * p.F + pp;
        const int axis = pp / p.F, jm = pp - axis * p.F;
        return axis * 2 * p.F + s * p.F + jm;
    }
    if (p.ndim == 1 && p.include_t && k == 2 * npairs) return 0;
    return k == p.widths[0] ? -1 : -2;
}

// NDIM (1 or 3) and ACT (hy_act) are template parameters, and FAST1D marks
// a 1-D length that is a power of two with every j t below 2^31 (the phase
// is then a mask and the angle an exact scaling): each instance holds only
// its own encoding and activation code.
template <int NDIM, int ACT, bool FAST1D>
__global__ void __launch_bounds__(NT, 2) filter_gen_tc2_kernel(const GenParams p) {
    extern __shared__ __align__(16) unsigned char sm2_raw[];
    uint8_t *tcb = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm2_raw) + 1023) & ~uintptr_t(1023));
    const int kpad = p.t_kpad, hpad = p.t_hpad, npad = p.t_npad;
    // A hi/lo: 128 position rows (the encodings, then the hidden outputs);
    // B0 hi/lo: hpad unit rows; B1 hi/lo: npad output rows of the slice
    uint8_t *a_hi = tcb, *a_lo = tcb + TP * TC_ROW;
    uint8_t *b0_hi = a_lo + TP * TC_ROW, *b0_lo = b0_hi + hpad * TC_ROW;
    uint8_t *b1_hi = b0_lo + hpad * TC_ROW, *b1_lo = b1_hi + npad * TC_ROW;
    float *bias1 = reinterpret_cast<float *>(b1_lo + npad * TC_ROW);   // output bias (0 when folded)
    float *al1 = bias1 + npad;                                         // decay rate x log2 e
    int *pdesc = reinterpret_cast<int *>(al1 + npad);                  // 3-D pair: axis | j << 2
    float2 *phase = reinterpret_cast<float2 *>(pdesc + 32);            // 3-D: (cos, sin)(pi m / g)
    __shared__ uint32_t s_tmem;
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int set = blockIdx.y;
    const int K0 = p.widths[0], H = p.widths[1], nout = p.widths[2];
    const int npairs = NDIM == 1 ? p.F : 3 * p.F;
    const int obase = blockIdx.z * p.t_slice;
    const int oend = min(nout, obase + p.t_slice);
    const int64_t ntiles = (p.npos + TP - 1) / TP;
    const bool film = p.gamma != nullptr;
    const bool fold_b1 = H < hpad;

    if (warp == 0) tc::tmem_alloc(&s_tmem, p.t_cols);
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    auto put_row = [&](uint8_t *hi, uint8_t *lo, int r, int c, const float (&v)[8]) {
        uint4 h4, l4;
        split_h2(v[0], v[1], h4.x, l4.x);
        split_h2(v[2], v[3], h4.y, l4.y);
        split_h2(v[4], v[5], h4.z, l4.z);
        split_h2(v[6], v[7], h4.w, l4.w);
        const uint32_t off = sw128_chunk(r, c);
        *reinterpret_cast<uint4 *>(hi + off) = h4;
        *reinterpret_cast<uint4 *>(lo + off) = l4;
    };
    // B0: row u = (1 + gamma_u) omega_u W0[u][feature(k)]; the constant
    // column omega_u ((1 + gamma_u) b0_u + beta_u); zero rows past H
    for (int idx = tid; idx < hpad * (kpad / 8); idx += NT) {
        const int u = idx / (kpad / 8), c = idx - u * (kpad / 8);
        float v[8];
        float sc = 0.f, bias = 0.f;
        if (u < H) {
            const float gm = film ? 1.f + __ldg(p.gamma + (int64_t)set * H + u) : 1.f;
            const float bt = film ? __ldg(p.beta + (int64_t)set * H + u) : 0.f;
            const float om = p.om[0] ? __ldg(p.om[0] + u) : 1.f;
            sc = gm * om;
            bias = om * fmaf(gm, __ldg(p.b[0] + u), bt);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int f = tc2_feature_of_column(p, 8 * c + j, npairs);
            v[j] = u >= H ? 0.f : (f >= 0 ? sc * __ldg(p.W[0] + (int64_t)u * K0 + f) : (f == -1 ? bias : 0.f));
        }
        put_row(b0_hi, b0_lo, u, c, v);
    }
    // B1: row o = W1[obase + o][k] for k < H, the output bias in column H
    // when it is free; zero rows past the slice
    for (int idx = tid; idx < npad * (hpad / 8); idx += NT) {
        const int o = idx / (hpad / 8), c = idx - o * (hpad / 8);
        const bool live = obase + o < oend;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = 8 * c + j;
            v[j] = !live ? 0.f
                         : (k < H ? __ldg(p.W[1] + (int64_t)(obase + o) * H + k)
                                  : (k == H ? __ldg(p.b[1] + obase + o) : 0.f));
        }
        put_row(b1_hi, b1_lo, o, c, v);
    }
    for (int o = tid; o < npad; o += NT) {
        const bool live = obase + o < oend;
        bias1[o] = (live && !fold_b1) ? __ldg(p.b[1] + obase + o) : 0.f;
        al1[o] = live ? __ldg(p.alpha + obase + o) * kLog2e : 0.f;
    }
    if constexpr (NDIM == 3) {
        for (int pp = tid; pp < npairs; pp += NT) pdesc[pp] = (pp / p.F) | ((pp % p.F + 1) << 2);
        for (int m = tid; m < 2 * p.g; m += NT) {
            float sn, cs;
            sincospif((float)m / (float)p.g, &sn, &cs);
            phase[m] = make_float2(cs, sn);
        }
    }
    fence_proxy_async_smem();                  // B0 and B1 are read by the tensor cores
    tc::fence_before();
    const uint32_t idesc0 = tc::idesc_f16(128, hpad, false);
    const uint32_t idesc1 = tc::idesc_f16(128, npad, false);
    uint32_t phase_bit = 0;
    // D[tmem + dcol] = A B^T with hi.hi + hi.lo + lo.hi; thread 0 issues and waits
    auto run_mma = [&](const uint8_t *Bhi, const uint8_t *Blo, uint32_t idesc, uint32_t dcol, int ksteps) {
        if (tid == 0) {
            tc::fence_after();
            bool first = true;
            for (int term = 0; term < 3; ++term) {
                const uint64_t ad = tc::desc_k_sw128(smem_u32(term == 2 ? a_lo : a_hi));
                const uint64_t bd = tc::desc_k_sw128(smem_u32(term == 1 ? Blo : Bhi));
                for (int ks = 0; ks < ksteps; ++ks) {
                    tc::mma_f16(s_tmem + dcol, ad + 2 * ks, bd + 2 * ks, idesc, first ? 0u : 1u);
                    first = false;
                }
            }
            tc::commit(&s_bar);
            if (!mbar_wait_sleep(&s_bar, phase_bit)) {
                record_fault(p.fault, HY_FAULT_FILTER_MMA);
                s_abort = 1;
            }
        }
        phase_bit ^= 1;
        __syncthreads();
        tc::fence_after();
    };
    const int q4 = warp & 3, hc = warp >> 2;
    const int pos = 32 * q4 + lane;            // this thread's position in the tile (its TMEM lane)
    const uint32_t trow = s_tmem + ((uint32_t)(32 * q4) << 16);
    const bool narrow = p.L * (int64_t)(p.F + 1) < (1LL << 31) && p.L <= (1 << 24);
    const float Lf = (float)p.L, invL = 1.f / Lf;   // exact when L is a power of two
    for (int64_t bt = blockIdx.x; bt < ntiles; bt += gridDim.x) {
        __syncthreads();                       // operands / TMEM of the previous tile released
        tc::fence_after();
        if (s_abort) break;                    // uniform: read between two barriers
        const int64_t qq = bt * TP + pos;
        const bool in = qq < p.npos;
        // ---- window argument and validity of the position; its signed
        //      offsets (3-D) for the encoding
        int r0 = 0, r1 = 0, r2 = 0;
        float nrm;
        bool valid = in;
        if constexpr (NDIM == 3) {
            const int S = p.S, ls = p.log_s;
            r0 = signed_off((int)(qq >> (2 * ls)) & (S - 1), S);
            r1 = signed_off((int)(qq >> ls) & (S - 1), S);
            r2 = signed_off((int)qq & (S - 1), S);
            valid = in && (p.circular || ((abs(r0) < p.g) && (abs(r1) < p.g) && (abs(r2) < p.g)));
            nrm = sqrtf((float)(r0 * r0 + r1 * r1 + r2 * r2)) / (float)p.g;
        } else {
            if constexpr (FAST1D) nrm = (float)qq * invL;
            else nrm = narrow ? __fdiv_rn((float)qq, Lf) : (float)((double)qq / (double)p.L);
        }
        // ---- encoding into A: the two warps of a lane quadrant take
        //      alternate 16-byte chunks (4 column pairs) of the row
        for (int c = hc; c < kpad / 8; c += 2) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pp = 4 * c + q;
                float cs, sn;
                if (pp < npairs) {
                    if constexpr (NDIM == 3) {
                        const int d = pdesc[pp];
                        const int ax = d & 3;
                        const int rv = ax == 0 ? r0 : (ax == 1 ? r1 : r2);
                        const float2 ph = phase[((d >> 2) * rv) & (2 * p.g - 1)];   // angle pi j r / g
                        cs = ph.x;
                        sn = ph.y;
                    } else {
                        const int j = pp + 1;
                        float arg;
                        if constexpr (FAST1D) {
                            const unsigned jt = (unsigned)(j * (int)qq);
                            arg = (float)(2u * (jt & (unsigned)(p.L - 1))) * invL;
                        } else if (narrow) {
                            const unsigned jt = (unsigned)(j * (int)qq);
                            arg = __fdiv_rn((float)(2u * (jt % (unsigned)p.L)), Lf);
                        } else {
                            const int64_t r = ((int64_t)j * qq) % p.L;
                            arg = (float)(2.0 * (double)r / (double)p.L);
                        }
                        sincospif(arg, &sn, &cs);        // angle 2 pi (j t mod L) / L
                    }
                } else {
                    const int k = 2 * pp;
                    const int kt = (NDIM == 1 && p.include_t) ? 2 * npairs : -1;
                    cs = k == kt ? nrm : (k == K0 ? 1.f : 0.f);
                    sn = k + 1 == kt ? nrm : (k + 1 == K0 ? 1.f : 0.f);
                }
                v[2 * q] = cs;
                v[2 * q + 1] = sn;
            }
            put_row(a_hi, a_lo, pos, c, v);
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---- first layer: the activation's argument per unit, TMEM columns 0 .. hpad-1
        run_mma(b0_hi, b0_lo, idesc0, 0u, kpad / 16);
        if (s_abort) break;                    // uniform: set before run_mma's barrier
        // ---- activation of this warp's half of the units, written over A
        {
            const int ub = hc * (hpad / 2), ue = ub + hpad / 2;
            uint32_t x[4][8];
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8)
                if (ub + 8 * g8 < ue) tc::tmem_ld8(trow + (uint32_t)(ub + 8 * g8), x[g8]);
            tc::tmem_wait_ld();
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                const int u0 = ub + 8 * g8;
                if (u0 >= ue) break;
                float a[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    float xv = __uint_as_float(x[g8][j]);
                    if constexpr (ACT == HY_ACT_SILU) xv = xv * rcp_fast(1.f + ex2_fast(-kLog2e * xv));
                    else if constexpr (ACT == HY_ACT_SINE) xv = sinf(xv);
                    a[j] = xv;
                }
                if (fold_b1 && u0 == (H & ~7)) {
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (u0 + j == H) a[j] = 1.f;   // the constant column of the output bias
                }
                put_row(a_hi, a_lo, pos, u0 / 8, a);
            }
        }
        tc::fence_before();
        fence_proxy_async_smem();
        __syncthreads();
        // ---- last layer: the slice's outputs, TMEM columns 128 ..
        run_mma(b1_hi, b1_lo, idesc1, TC2_OUT_COL, hpad / 16);
        {
            float nr = nrm;
            if (p.window == HY_WIN_GAUSS) nr *= nr;
            const float nrn = valid ? -nr : 0.f;
            for (int c0 = 16 * hc; c0 < npad; c0 += 32) {
                __syncwarp();                  // tcgen05.ld is warp-wide
                uint32_t v[16];
                tc::tmem_ld16(trow + TC2_OUT_COL + (uint32_t)c0, v);
                tc::tmem_wait_ld();
                float y[16];
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(al1 + c0 + 4 * j4);
                    const float4 b4 = *reinterpret_cast<const float4 *>(bias1 + c0 + 4 * j4);
                    y[4 * j4 + 0] = (__uint_as_float(v[4 * j4 + 0]) + b4.x) * ex2_fast(a4.x * nrn);
                    y[4 * j4 + 1] = (__uint_as_float(v[4 * j4 + 1]) + b4.y) * ex2_fast(a4.y * nrn);
                    y[4 * j4 + 2] = (__uint_as_float(v[4 * j4 + 2]) + b4.z) * ex2_fast(a4.z * nrn);
                    y[4 * j4 + 3] = (__uint_as_float(v[4 * j4 + 3]) + b4.w) * ex2_fast(a4.w * nrn);
                }
                const int ob = obase + c0;
                float *dst = p.h + ((int64_t)set * nout + ob) * p.npos + qq;
                if (in && ob + 16 <= oend) {
#pragma unroll
                    for (int j = 0; j < 16; ++j, dst += p.npos) *dst = valid ? y[j] : 0.f;
                } else if (in) {
#pragma unroll
                    for (int j = 0; j < 16; ++j, dst += p.npos)
                        if (ob + j < oend) *dst = valid ? y[j] : 0.f;
                }
            }
        }
        tc::fence_before();
    }
    // no MMA may still be running when TMEM is freed (all were waited on;
    // this covers one whose wait gave up)
    if (tid == 0) {
        tc::commit(&s_bar);
        if (!mbar_wait_sleep(&s_bar, phase_bit)) record_fault(p.fault, HY_FAULT_FILTER_MMA);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    __syncwarp();
    if (warp == 0) tc::tmem_free(s_tmem, p.t_cols);
}

// ----------------------------------------------------------------------------
// All three layers on the tensor cores (two hidden layers of <= 64 units,
// input width <= 127), for filter sets with fewer 128-position tiles than
// SMs and many outputs: workload 2's 768 outputs over 8192 positions are 64
// tiles, too few to spread one tile per CTA over the SMs in one pass of the
// outputs.  A CTA takes one tile and the output slices blockIdx.z,
// + gridDim.z, ... (128 outputs each): it encodes the tile into the first
// operand (fp16 hi/lo, up to two 64-column atoms; columns as in
// filter_gen_tc2_kernel), runs the first layer (FiLM, sine frequencies and
// bias folded into the held weights), activates into the operand, runs the
// second layer (sine frequencies folded, bias added before the
// activation), activates again, and then for each slice loads the slice's
// last-layer weights, runs the last layer and stores with the decay window.
// The hidden layers are computed once per tile and CTA.
// ----------------------------------------------------------------------------
template <int NDIM, int ACT, bool FAST1D>
__global__ void __launch_bounds__(NT, 1) filter_gen_tc3_kernel(const GenParams p) {
    extern __shared__ __align__(16) unsigned char sm3_raw[];
    uint8_t *tcb = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm3_raw) + 1023) & ~uintptr_t(1023));
    const int kpad = p.t_kpad, h1p = p.t_hpad, h2p = p.t_h2pad, npad = p.t_npad;
    const int ka = (kpad + 63) / 64;           // 64-column atoms of the first operand
    // A hi/lo: ka atoms of 128 position rows; B0: ka atoms of h1p rows; B1:
    // h2p rows; B2: npad rows of the current slice
    uint8_t *a_hi = tcb, *a_lo = a_hi + ka * TP * TC_ROW;
    uint8_t *b0_hi = a_lo + ka * TP * TC_ROW, *b0_lo = b0_hi + ka * h1p * TC_ROW;
    uint8_t *b1_hi = b0_lo + ka * h1p * TC_ROW, *b1_lo = b1_hi + h2p * TC_ROW;
    uint8_t *b2_hi = b1_lo + h2p * TC_ROW, *b2_lo = b2_hi + npad * TC_ROW;
    float *bias1 = reinterpret_cast<float *>(b2_lo + npad * TC_ROW);   // second hidden layer: omega b
    float *bias2 = bias1 + 64;                                         // slice's output bias
    float *al2 = bias2 + npad;                                         // slice's decay rate x log2 e
    int *pdesc = reinterpret_cast<int *>(al2 + npad);                  // 3-D pair: axis | j << 2
    float2 *phase = reinterpret_cast<float2 *>(pdesc + 64);            // 3-D: (cos, sin)(pi m / g)
    __shared__ uint32_t s_tmem;
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int set = blockIdx.y;
    const int K0 = p.widths[0], H1 = p.widths[1], H2 = p.widths[2], nout = p.widths[3];
    const int npairs = NDIM == 1 ? p.F : 3 * p.F;
    const int64_t ntiles = (p.npos + TP - 1) / TP;
    const bool film = p.gamma != nullptr;

    if (warp == 0) tc::tmem_alloc(&s_tmem, p.t_cols);
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    // 16-byte chunk c (8 columns) of row r of an operand of `rows` rows
    auto put_row = [&](uint8_t *hi, uint8_t *lo, int rows, int r, int c, const float (&v)[8]) {
        uint4 h4, l4;
        split_h2(v[0], v[1], h4.x, l4.x);
        split_h2(v[2], v[3], h4.y, l4.y);
        split_h2(v[4], v[5], h4.z, l4.z);
        split_h2(v[6], v[7], h4.w, l4.w);
        const uint32_t off = (uint32_t)((c >> 3) * rows * TC_ROW) + sw128_chunk(r, c & 7);
        *reinterpret_cast<uint4 *>(hi + off) = h4;
        *reinterpret_cast<uint4 *>(lo + off) = l4;
    };
    // B0: row u = (1 + gamma_u) omega_u W0[u][feature(k)]; the constant
    // column omega_u ((1 + gamma_u) b0_u + beta_u); zero rows past H1
    for (int idx = tid; idx < h1p * (kpad / 8); idx += NT) {
        const int u = idx / (kpad / 8), c = idx - u * (kpad / 8);
        float v[8];
        float sc = 0.f, bias = 0.f;
        if (u < H1) {
            const float gm = film ? 1.f + __ldg(p.gamma + (int64_t)set * H1 + u) : 1.f;
            const float bt = film ? __ldg(p.beta + (int64_t)set * H1 + u) : 0.f;
            const float om = p.om[0] ? __ldg(p.om[0] + u) : 1.f;
            sc = gm * om;
            bias = om * fmaf(gm, __ldg(p.b[0] + u), bt);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int f = tc2_feature_of_column(p, 8 * c + j, npairs);
            v[j] = u >= H1 ? 0.f : (f >= 0 ? sc * __ldg(p.W[0] + (int64_t)u * K0 + f) : (f == -1 ? bias : 0.f));
        }
        put_row(b0_hi, b0_lo, h1p, u, c, v);
    }
    // B1: row u = omega_u W1[u][k] (k < H1); its bias omega_u b1_u is added
    // before the activation
    for (int idx = tid; idx < h2p * (h1p / 8); idx += NT) {
        const int u = idx / (h1p / 8), c = idx - u * (h1p / 8);
        const float om = (u < H2 && p.om[1]) ? __ldg(p.om[1] + u) : 1.f;
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int k = 8 * c + j;
            v[j] = (u < H2 && k < H1) ? om * __ldg(p.W[1] + (int64_t)u * H1 + k) : 0.f;
        }
        put_row(b1_hi, b1_lo, h2p, u, c, v);
    }
    for (int u = tid; u < 64; u += NT) {
        const float om = (u < H2 && p.om[1]) ? __ldg(p.om[1] + u) : 1.f;
        bias1[u] = u < H2 ? om * __ldg(p.b[1] + u) : 0.f;
    }
    if constexpr (NDIM == 3) {
        for (int pp = tid; pp < npairs; pp += NT) pdesc[pp] = (pp / p.F) | ((pp % p.F + 1) << 2);
        for (int m = tid; m < 2 * p.g; m += NT) {
            float sn, cs;
            sincospif((float)m / (float)p.g, &sn, &cs);
            phase[m] = make_float2(cs, sn);
        }
    }
    // B2 and the per-output rows of slice sl
    auto load_slice = [&](int sl) {
        const int obase = sl * p.t_slice, oend = min(nout, obase + p.t_slice);
        for (int idx = tid; idx < npad * (h2p / 8); idx += NT) {
            const int o = idx / (h2p / 8), c = idx - o * (h2p / 8);
            const bool live = obase + o < oend;
            float v[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = 8 * c + j;
                v[j] = (live && k < H2) ? __ldg(p.W[2] + (int64_t)(obase + o) * H2 + k) : 0.f;
            }
            put_row(b2_hi, b2_lo, npad, o, c, v);
        }
        for (int o = tid; o < npad; o += NT) {
            const bool live = obase + o < oend;
            bias2[o] = live ? __ldg(p.b[2] + obase + o) : 0.f;
            al2[o] = live ? __ldg(p.alpha + obase + o) * kLog2e : 0.f;
        }
    };
    fence_proxy_async_smem();                  // B0 and B1 are read by the tensor cores
    tc::fence_before();
    uint32_t phase_bit = 0;
    // D[tmem + dcol] = A B^T over ksteps of 16 columns (atoms of 4 steps;
    // A atoms TP rows apart, B atoms b_rows rows apart): hi.hi + hi.lo + lo.hi
    auto run_mma = [&](const uint8_t *Bhi, const uint8_t *Blo, int b_rows, uint32_t idesc, uint32_t dcol,
                       int ksteps) {
        if (tid == 0) {
            tc::fence_after();
            bool first = true;
            for (int term = 0; term < 3; ++term) {
                const uint8_t *A = term == 2 ? a_lo : a_hi;
                const uint8_t *Bm = term == 1 ? Blo : Bhi;
                for (int ks = 0; ks < ksteps; ++ks) {
                    const uint64_t ad = tc::desc_k_sw128(smem_u32(A + (ks >> 2) * TP * TC_ROW)) + 2 * (ks & 3);
                    const uint64_t bd = tc::desc_k_sw128(smem_u32(Bm + (ks >> 2) * b_rows * TC_ROW)) + 2 * (ks & 3);
                    tc::mma_f16(s_tmem + dcol, ad, bd, idesc, first ? 0u : 1u);
                    first = false;
                }
            }
            tc::commit(&s_bar);
            if (!mbar_wait_sleep(&s_bar, phase_bit)) {
                record_fault(p.fault, HY_FAULT_FILTER_MMA);
                s_abort = 1;
            }
        }
        phase_bit ^= 1;
        __syncthreads();
        tc::fence_after();
    };
    // activation of this warp's half of the units of TMEM columns dcol ..
    // (plus bias[u] when given) into chunk columns of the first operand
    auto activate = [&](uint32_t trow, uint32_t dcol, int hp, int Hn, const float *bias, int pos, int hc) {
        const int ub = hc * (hp / 2), ue = ub + hp / 2;
        uint32_t x[4][8];
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8)
            if (ub + 8 * g8 < ue) tc::tmem_ld8(trow + dcol + (uint32_t)(ub + 8 * g8), x[g8]);
        tc::tmem_wait_ld();
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
            const int u0 = ub + 8 * g8;
            if (u0 >= ue) break;
            float a[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float xv = __uint_as_float(x[g8][j]);
                if (bias) xv += bias[u0 + j];
                if constexpr (ACT == HY_ACT_SILU) xv = xv * rcp_fast(1.f + ex2_fast(-kLog2e * xv));
                else if constexpr (ACT == HY_ACT_SINE) xv = sinf(xv);
                a[j] = u0 + j < Hn ? xv : 0.f;
            }
            put_row(a_hi, a_lo, TP, pos, u0 / 8, a);
        }
    };
    const uint32_t idesc0 = tc::idesc_f16(128, h1p, false);
    const uint32_t idesc1 = tc::idesc_f16(128, h2p, false);
    const uint32_t idesc2 = tc::idesc_f16(128, npad, false);
    constexpr uint32_t D1_COL = 64, D2_COL = 128;
    const int q4 = warp & 3, hc = warp >> 2;
    const int pos = 32 * q4 + lane;            // this thread's position in the tile (its TMEM lane)
    const uint32_t trow = s_tmem + ((uint32_t)(32 * q4) << 16);
    const bool narrow = p.L * (int64_t)(p.F + 1) < (1LL << 31) && p.L <= (1 << 24);
    const float Lf = (float)p.L, invL = 1.f / Lf;   // exact when L is a power of two
    int cur_slice = -1;
    for (int64_t bt = blockIdx.x; bt < ntiles; bt += gridDim.x) {
        __syncthreads();                       // operands / TMEM of the previous tile released
        tc::fence_after();
        if (s_abort) break;                    // uniform: read between two barriers
        const int64_t qq = bt * TP + pos;
        const bool in = qq < p.npos;
        int r0 = 0, r1 = 0, r2 = 0;
        float nrm;
        bool valid = in;
        if constexpr (NDIM == 3) {
            const int S = p.S, ls = p.log_s;
            r0 = signed_off((int)(qq >> (2 * ls)) & (S - 1), S);
            r1 = signed_off((int)(qq >> ls) & (S - 1), S);
            r2 = signed_off((int)qq & (S - 1), S);
            valid = in && (p.circular || ((abs(r0) < p.g) && (abs(r1) < p.g) && (abs(r2) < p.g)));
            nrm = sqrtf((float)(r0 * r0 + r1 * r1 + r2 * r2)) / (float)p.g;
        } else {
            if constexpr (FAST1D) nrm = (float)qq * invL;
            else nrm = narrow ? __fdiv_rn((float)qq, Lf) : (float)((double)qq / (double)p.L);
        }
        // ---- encoding into A (up to two atoms): the two warps of a lane
        //      quadrant take alternate 16-byte chunks
        for (int c = hc; c < kpad / 8; c += 2) {
            float v[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int pp = 4 * c + q;
                float cs, sn;
                if (pp < npairs) {
                    if constexpr (NDIM == 3) {
                        const int d = pdesc[pp];
                        const int ax = d & 3;
                        const int rv = ax == 0 ? r0 : (ax == 1 ? r1 : r2);
                        const float2 ph = phase[((d >> 2) * rv) & (2 * p.g - 1)];
                        cs = ph.x;
                        sn = ph.y;
                    } else {
                        const int j = pp + 1;
                        float arg;
                        if constexpr (FAST1D) {
                            const unsigned jt = (unsigned)(j * (int)qq);
                            arg = (float)(2u * (jt & (unsigned)(p.L - 1))) * invL;
                        } else if (narrow) {
                            const unsigned jt = (unsigned)(j * (int)qq);
                            arg = __fdiv_rn((float)(2u * (jt % (unsigned)p.L)), Lf);
                        } else {
                            const int64_t r = ((int64_t)j * qq) % p.L;
                            arg = (float)(2.0 * (double)r / (double)p.L);
                        }
                        sincospif(arg, &sn, &cs);    // angle 2 pi (j t mod L) / L
                    }
                } else {
                    const int kc = 2 * pp;
                    const int kt = (NDIM == 1 && p.include_t) ? 2 * npairs : -1;
                    cs = kc == kt ? nrm : (kc == K0 ? 1.f : 0.f);
                    sn = kc + 1 == kt ? nrm : (kc + 1 == K0 ? 1.f : 0.f);
                }
                v[2 * q] = cs;
                v[2 * q + 1] = sn;
            }
            put_row(a_hi, a_lo, TP, pos, c, v);
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---- first hidden layer (its argument: biases and FiLM folded)
        run_mma(b0_hi, b0_lo, h1p, idesc0, 0u, kpad / 16);
        if (s_abort) break;
        activate(trow, 0u, h1p, H1, nullptr, pos, hc);
        tc::fence_before();
        fence_proxy_async_smem();
        __syncthreads();
        // ---- second hidden layer
        run_mma(b1_hi, b1_lo, h2p, idesc1, D1_COL, h1p / 16);
        if (s_abort) break;
        activate(trow, D1_COL, h2p, H2, bias1, pos, hc);
        tc::fence_before();
        fence_proxy_async_smem();
        // ---- the output slices of this CTA
        for (int sl = blockIdx.z; sl < p.t_nslices; sl += gridDim.z) {
            const int obase = sl * p.t_slice;
            const int oend = min(nout, obase + p.t_slice);
            __syncthreads();                   // A written; the last MMA and TMEM reads done
            if (sl != cur_slice) {
                load_slice(sl);
                cur_slice = sl;
                fence_proxy_async_smem();
                __syncthreads();
            }
            run_mma(b2_hi, b2_lo, npad, idesc2, D2_COL, h2p / 16);
            if (s_abort) break;
            float nr = nrm;
            if (p.window == HY_WIN_GAUSS) nr *= nr;
            const float nrn = valid ? -nr : 0.f;
            for (int c0 = 16 * hc; c0 < npad; c0 += 32) {
                __syncwarp();                  // tcgen05.ld is warp-wide
                uint32_t v[16];
                tc::tmem_ld16(trow + D2_COL + (uint32_t)c0, v);
                tc::tmem_wait_ld();
                float y[16];
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(al2 + c0 + 4 * j4);
                    const float4 b4 = *reinterpret_cast<const float4 *>(bias2 + c0 + 4 * j4);
                    y[4 * j4 + 0] = (__uint_as_float(v[4 * j4 + 0]) + b4.x) * ex2_fast(a4.x * nrn);
                    y[4 * j4 + 1] = (__uint_as_float(v[4 * j4 + 1]) + b4.y) * ex2_fast(a4.y * nrn);
                    y[4 * j4 + 2] = (__uint_as_float(v[4 * j4 + 2]) + b4.z) * ex2_fast(a4.z * nrn);
                    y[4 * j4 + 3] = (__uint_as_float(v[4 * j4 + 3]) + b4.w) * ex2_fast(a4.w * nrn);
                }
                const int ob = obase + c0;
                float *dst = p.h + ((int64_t)set * nout + ob) * p.npos + qq;
                if (in && ob + 16 <= oend) {
#pragma unroll
                    for (int j = 0; j < 16; ++j, dst += p.npos) *dst = valid ? y[j] : 0.f;
                } else if (in) {
#pragma unroll
                    for (int j = 0; j < 16; ++j, dst += p.npos)
                        if (ob + j < oend) *dst = valid ? y[j] : 0.f;
                }
            }
            tc::fence_before();
        }
        if (s_abort) break;
    }
    // no MMA may still be running when TMEM is freed (all were waited on;
    // this covers one whose wait gave up)
    if (tid == 0) {
        tc::commit(&s_bar);
        if (!mbar_wait_sleep(&s_bar, phase_bit)) record_fault(p.fault, HY_FAULT_FILTER_MMA);
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    __syncwarp();
    if (warp == 0) tc::tmem_free(s_tmem, p.t_cols);
}

// Engine of the layers: HYENA_FILTER_ENGINE=simt keeps them on the FP32
// pipes, =tensor_last puts only the last layer on the tensor cores, =tensor
// (or unset) both layers of a one-hidden-layer MLP where that kernel applies,
// else the last layer.
int filter_engine() {
    const char *e = std::getenv("HYENA_FILTER_ENGINE");
    if (e && std::strcmp(e, "simt") == 0) return 0;
    if (e && std::strcmp(e, "tensor_last") == 0) return 3;
    if (e && std::strcmp(e, "tensor") == 0) return 2;
    return 1;
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
    // Both layers on the tensor cores: one hidden layer, input width <= 63
    // (a free column for the bias), hidden width <= 64, output slices of
    // <= 128 (two CTAs of 256 TMEM columns per SM), at least one 128-position
    // tile per SM.
    {
        GenParams q = p;
        const int nlast = q.widths[q.nl];
        const int64_t ntiles = (q.npos + TP - 1) / TP;
        const int eng = filter_engine();
        if ((eng == 1 || eng == 2) && q.nl == 2 && q.widths[0] <= 63 && q.widths[1] <= 64 &&
            ntiles * d.n_sets >= sms) {
            q.t_slice = nlast > 128 ? 128 : nlast;
            const int nslices = (nlast + q.t_slice - 1) / q.t_slice;
            q.t_kpad = (q.widths[0] + 1 + 15) & ~15;
            q.t_hpad = (q.widths[1] + 15) & ~15;
            q.t_npad = (q.t_slice + 15) & ~15;
            q.t_cols = 32;
            while ((int)q.t_cols < (int)TC2_OUT_COL + q.t_npad) q.t_cols <<= 1;
            q.fault = device_fault_word();
            if (!q.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
            size_t smem = 1024 + (size_t)2 * TC_ROW * (TP + q.t_hpad + q.t_npad) +
                          sizeof(float) * (2 * (size_t)q.t_npad + 32) + (q.ndim == 3 ? (size_t)16 * q.g : 0);
            const int fit = 512 / (int)q.t_cols;
            const size_t floor_smem = (size_t)233472 / (size_t)(fit + 1) + 1024;
            if (fit < 8 && smem < floor_smem) smem = floor_smem;
            if (nslices <= 65535 && smem <= (size_t)227 * 1024) {
                void (*kern)(const GenParams) = nullptr;
                const bool fast1d = q.L * (int64_t)(q.F + 1) < (1LL << 31) && q.L <= (1 << 24) && (q.L & (q.L - 1)) == 0;
                if (q.ndim == 3)
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc2_kernel<3, HY_ACT_SILU, false>
                         : q.act == HY_ACT_SINE ? filter_gen_tc2_kernel<3, HY_ACT_SINE, false>
                                                : filter_gen_tc2_kernel<3, HY_ACT_IDENTITY, false>;
                else if (fast1d)
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc2_kernel<1, HY_ACT_SILU, true>
                         : q.act == HY_ACT_SINE ? filter_gen_tc2_kernel<1, HY_ACT_SINE, true>
                                                : filter_gen_tc2_kernel<1, HY_ACT_IDENTITY, true>;
                else
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc2_kernel<1, HY_ACT_SILU, false>
                         : q.act == HY_ACT_SINE ? filter_gen_tc2_kernel<1, HY_ACT_SINE, false>
                                                : filter_gen_tc2_kernel<1, HY_ACT_IDENTITY, false>;
                cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return set_cuda_error("filter_gen two-layer smem attribute", e);
                e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
                if (e != cudaSuccess) return set_cuda_error("filter_gen carve-out attribute", e);
                int per_sm = (int)((size_t)233472 / (smem + 1024));
                if (per_sm > 2) per_sm = 2;
                if (per_sm > fit) per_sm = fit;
                if (per_sm < 1) per_sm = 1;
                int64_t per_set = ((int64_t)per_sm * sms + (int64_t)d.n_sets * nslices - 1) / ((int64_t)d.n_sets * nslices);
                if (per_set > ntiles) per_set = ntiles;
                dim3 grid((unsigned)per_set, (unsigned)d.n_sets, (unsigned)nslices);
                kern<<<grid, NT, smem, s>>>(q);
                return check_launch("filter_gen (two tensor-core layers) launch");
            }
        }
    }
    // All three layers on the tensor cores: two hidden layers of <= 64 units,
    // input width <= 127, fewer 128-position tiles than SMs and at least 256
    // outputs.  One CTA per (tile, set, slice group): grid z splits the
    // 128-output slices so that the CTAs about fill the SMs.
    {
        GenParams q = p;
        const int64_t ntiles = (q.npos + TP - 1) / TP;
        const int eng = filter_engine();
        if ((eng == 1 || eng == 2) && q.nl == 3 && q.widths[0] <= 127 && q.widths[1] <= 64 && q.widths[2] <= 64 &&
            q.widths[3] >= 256 && ntiles * d.n_sets < sms) {
            const int nout = q.widths[3];
            q.t_slice = 128;
            q.t_nslices = (nout + 127) / 128;
            int zsplit = (int)(sms / (ntiles * d.n_sets));
            if (zsplit < 1) zsplit = 1;
            if (zsplit > q.t_nslices) zsplit = q.t_nslices;
            q.t_kpad = (q.widths[0] + 1 + 15) & ~15;
            q.t_hpad = (q.widths[1] + 15) & ~15;
            q.t_h2pad = (q.widths[2] + 15) & ~15;
            q.t_npad = 128;
            q.t_cols = 256;
            q.fault = device_fault_word();
            if (!q.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
            const int ka = (q.t_kpad + 63) / 64;
            const size_t smem = 1024 + (size_t)2 * TC_ROW * (ka * TP + ka * q.t_hpad + q.t_h2pad + q.t_npad) +
                                sizeof(float) * (64 + 2 * (size_t)q.t_npad) + sizeof(int) * 64 +
                                (q.ndim == 3 ? (size_t)16 * q.g : 0);
            if (smem <= (size_t)227 * 1024) {
                void (*kern)(const GenParams) = nullptr;
                const bool fast1d = q.L * (int64_t)(q.F + 1) < (1LL << 31) && q.L <= (1 << 24) && (q.L & (q.L - 1)) == 0;
                if (q.ndim == 3)
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc3_kernel<3, HY_ACT_SILU, false>
                         : q.act == HY_ACT_SINE ? filter_gen_tc3_kernel<3, HY_ACT_SINE, false>
                                                : filter_gen_tc3_kernel<3, HY_ACT_IDENTITY, false>;
                else if (fast1d)
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc3_kernel<1, HY_ACT_SILU, true>
                         : q.act == HY_ACT_SINE ? filter_gen_tc3_kernel<1, HY_ACT_SINE, true>
                                                : filter_gen_tc3_kernel<1, HY_ACT_IDENTITY, true>;
                else
                    kern = q.act == HY_ACT_SILU ? filter_gen_tc3_kernel<1, HY_ACT_SILU, false>
                         : q.act == HY_ACT_SINE ? filter_gen_tc3_kernel<1, HY_ACT_SINE, false>
                                                : filter_gen_tc3_kernel<1, HY_ACT_IDENTITY, false>;
                cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return set_cuda_error("filter_gen three-layer smem attribute", e);
                e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
                if (e != cudaSuccess) return set_cuda_error("filter_gen carve-out attribute", e);
                dim3 grid((unsigned)ntiles, (unsigned)d.n_sets, (unsigned)zsplit);
                kern<<<grid, NT, smem, s>>>(q);
                return check_launch("filter_gen (three tensor-core layers) launch");
            }
        }
    }
    // Tensor-core last layer: a hidden layer before it, K <= 128, at least one
    // (128-position tile, output slice) pair per SM.
    {
        GenParams q = p;
        const int Klast = q.widths[q.nl - 1];
        const int nlast = q.widths[q.nl];
        const int64_t ntiles = (q.npos + TP - 1) / TP;
        // more than 512 outputs: split over grid z in slices of 256 (each
        // slice recomputes the hidden layers).  With fewer position tiles than
        // SMs the FP32-pipe kernels stay: slicing the 768 outputs of an
        // 8192-position filter set over 64 tiles measured 2x slower than them.
        q.t_slice = nlast > 512 ? 256 : nlast;
        const int nslices = (nlast + q.t_slice - 1) / q.t_slice;
        if (filter_engine() > 0 && q.nl >= 2 && Klast <= 128 && nslices <= 64 && ntiles * d.n_sets >= sms) {
            const int64_t rfl = resident_layout(q, true);
            q.t_kpad = (Klast + 15) & ~15;
            q.t_katoms = (q.t_kpad + 63) / 64;
            q.t_npad = (q.t_slice + 15) & ~15;
            q.t_cols = 32;
            while ((int)q.t_cols < q.t_npad) q.t_cols <<= 1;
            q.fault = device_fault_word();
            if (!q.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
            size_t smem = sizeof(float) * ((size_t)2 * q.ka * P + (size_t)rfl) + 1024 +
                          (size_t)2 * q.t_katoms * TP * TC_ROW + (size_t)2 * q.t_katoms * q.t_npad * TC_ROW;
            // the CTAs that share an SM must fit its 512 TMEM columns: ask for
            // enough shared memory that no more of them can be resident
            const int fit = 512 / (int)q.t_cols;
            const size_t floor_smem = (size_t)233472 / (size_t)(fit + 1) + 1024;
            if (fit < 8 && smem < floor_smem) smem = floor_smem;
            if (smem <= (size_t)227 * 1024) {
                cudaError_t e = cudaFuncSetAttribute(filter_gen_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)smem);
                if (e != cudaSuccess) return set_cuda_error("filter_gen tensor-core smem attribute", e);
                e = cudaFuncSetAttribute(filter_gen_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
                if (e != cudaSuccess) return set_cuda_error("filter_gen carve-out attribute", e);
                // CTAs per SM from the shared memory they take (two at most: the
                // launch bounds give each thread 128 registers)
                int per_sm = (int)((size_t)233472 / (smem + 1024));
                if (per_sm > 2) per_sm = 2;
                if (per_sm > fit) per_sm = fit;
                if (per_sm < 1) per_sm = 1;
                int64_t per_set = ((int64_t)per_sm * sms + (int64_t)d.n_sets * nslices - 1) / ((int64_t)d.n_sets * nslices);
                if (per_set > ntiles) per_set = ntiles;
                dim3 grid((unsigned)per_set, (unsigned)d.n_sets, (unsigned)nslices);
                filter_gen_tc_kernel<<<grid, NT, smem, s>>>(q, rfl);
                return check_launch("filter_gen (tensor-core last layer) launch");
            }
        }
    }
    // Many position tiles per set, weights that fit in shared memory: keep
    // them resident in persistent CTAs instead of staging them per tile (only
    // with two CTAs per SM: with one, the FP32 pipes idle at every barrier and
    // the streaming kernel's two CTAs per SM are faster).
    {
        GenParams q = p;
        const int64_t rfl = resident_layout(q, false);
        const size_t rsmem = sizeof(float) * ((size_t)2 * q.ka * P + (size_t)rfl);
        if (nblk * d.n_sets >= (int64_t)8 * sms && rsmem <= (size_t)113 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(filter_gen_resident_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)rsmem);
            if (e != cudaSuccess) return set_cuda_error("filter_gen resident smem attribute", e);
            e = cudaFuncSetAttribute(filter_gen_resident_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
            if (e != cudaSuccess) return set_cuda_error("filter_gen carve-out attribute", e);
            int64_t per_set = ((int64_t)2 * sms + d.n_sets - 1) / d.n_sets;
            if (per_set > nblk) per_set = nblk;
            dim3 grid((unsigned)per_set, (unsigned)d.n_sets, 1);
            filter_gen_resident_kernel<<<grid, NT, rsmem, s>>>(q);
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
