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
#include "kernels.h"
#include "status.h"

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

// acc[a][c] = sum_k act[k][4tx + a] * wT[k][CPT*ty + c], k ascending.
template <int CPT>
__device__ __forceinline__ void tile_gemm(const float *act, const float *wT, int K, int tx, int ty,
                                          float (&acc)[4][CPT]) {
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
            const float4 wv = *reinterpret_cast<const float4 *>(wp + k * OTS + 4 * c4);
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
    const size_t smem = sizeof(float) * ((size_t)2 * p.ka * P + (size_t)2 * p.wbuf);
    cudaError_t e = cudaFuncSetAttribute(filter_gen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return set_cuda_error("filter_gen smem attribute", e);
    // split the last layer over grid z only when there are fewer CTAs than
    // SMs (each split recomputes the hidden layers)
    const int nout = d.widths[d.n_layers];
    const int64_t base = nblk * d.n_sets;
    int sms = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
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
