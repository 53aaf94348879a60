// filter_gen.cu -- fused implicit filter generator.
//
// [HN] 아키텍처 상세, step 2: h(t) = FFN(pos_enc(t)) · w(t), w(t) = e^{-αt};
// [ES] 어떻게 동작하나요?: a small MLP with sinusoidal features and an
// exponential decay window; [ND] 방법론: HyenaND: coordinate MLP on the N-D
// grid with FiLM conditioning per sample.
//
// One CTA owns P = 64 consecutive positions of one filter set.  It builds
// the positional encoding in shared memory and runs the hidden layers on the
// FP32 pipes: 64-output tiles, each an fp32 GEMM over K = layer input width
// accumulated as K outer products into a 4-position x 4-output register tile
// per thread (activations act[k][pos], one float4 read; weights wT[k][o],
// transposed while staged by cp.async, double-buffered across tiles).
// Hidden outputs get bias, FiLM and the activation and stay in shared memory.
//
// The last layer -- most of the MACs -- runs on the tcgen05 tensor cores.
// For each tile of 128 outputs, D[o][p] = Σ_k W[o][k] a[p][k] is a chain of
// M = 128, N = 64, K = 8 MMAs (kind::tf32) with the accumulator in tensor
// memory.  Each fp32 operand x is split into x_hi = x with its 13 low
// mantissa bits cleared and x_lo = the same of x - x_hi (exact), and the sum
// lo·hi + hi·lo + hi·hi keeps fp32-level accuracy (the dropped lo·lo term is
// below 2^-20 of the product).  Both operands sit in shared memory in the
// K-major, unswizzled core-matrix layout: a core matrix is 8 rows x 4 values
// (16 bytes per row), K chunks are 128 bytes apart and 8-row groups kpad*32
// bytes apart.  The last hidden layer writes its activations straight into
// that layout.  The epilogue reads the accumulator back with tcgen05.ld (one
// output row per thread, 32 positions per warp), adds the bias, applies the
// decay window and stores the rows to HBM.  Only when the grid has fewer
// CTAs than SMs is the last layer split over grid z (each split recomputes
// the small hidden layers).  The one wait on the tensor cores is bounded.
#include "bulk_copy.cuh"
#include "common.cuh"
#include "kernels.h"
#include "status.h"

namespace hy {

namespace {

constexpr int P = 64;           // positions per CTA (the MMA's N)
constexpr int NT = 256;         // threads: 16 position groups x 16 output groups
constexpr int CPT = 4;          // outputs per thread in a hidden tile
constexpr int OT = 16 * CPT;    // outputs per hidden tile
constexpr int OTS = OT + 4;     // wT row stride: = 4 (mod 32) keeps the staging stores conflict-free
constexpr int MAXW = 132;       // max layer input width
constexpr int MAXL = 4;
constexpr int NPAR = 4;         // per-output rows staged with a hidden tile: bias, gamma, beta, omega
constexpr int MT = 128;         // last-layer outputs per MMA tile (the MMA's M)
constexpr uint32_t TMEM_COLS = 64;   // the fp32 accumulator: 128 lanes x P columns

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
    int ka;                     // max hidden-layer input width (activation rows)
    int wbuf;                   // floats per hidden weight buffer
    int kpad;                   // last-layer K rounded up to a multiple of 8
    int u_floats;               // floats of the region shared by the hidden phase and the last-layer A operand
    int out_chunk;              // last-layer outputs per grid-z slice (multiple of MT)
    int vec_out;                // float4 stores of the output rows are aligned
    int vec_w;                  // last-layer weight rows can be read as float4
    float *h;
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

// ---- TF32 operand split and the UMMA operand layout
__device__ __forceinline__ float tf32_trunc(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }
// float index of the 16-byte chunk holding (row, k = 4 kc .. 4 kc + 3)
__device__ __forceinline__ int umma_chunk(int row, int kc, int kpad) {
    return (row >> 3) * (kpad * 8) + kc * 32 + (row & 7) * 4;
}
// stores the chunk v split into its hi and lo parts
__device__ __forceinline__ void store_split(float *hi, float *lo, int off, float4 v) {
    const float4 h = make_float4(tf32_trunc(v.x), tf32_trunc(v.y), tf32_trunc(v.z), tf32_trunc(v.w));
    const float4 l = make_float4(tf32_trunc(v.x - h.x), tf32_trunc(v.y - h.y), tf32_trunc(v.z - h.z),
                                 tf32_trunc(v.w - h.w));
    *reinterpret_cast<float4 *>(hi + off) = h;
    *reinterpret_cast<float4 *>(lo + off) = l;
}
// shared-memory matrix descriptor of a K-major, unswizzled operand starting
// at shared address `saddr`: leading offset 128 B (next K chunk), stride
// offset kpad*32 B (next 8-row group), descriptor version 1
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, int kpad) {
    return (uint64_t)((saddr >> 4) & 0x3fffu) | ((uint64_t)(128u >> 4) << 16) |
           ((uint64_t)(((uint32_t)kpad * 32u) >> 4) << 32) | ((uint64_t)1 << 46);
}
// instruction descriptor: D fp32, A and B tf32, both K-major, M = 128, N = P
constexpr uint32_t kInstrDesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(P >> 3) << 17) |
                                ((uint32_t)(MT >> 4) << 24);

__device__ __forceinline__ void umma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kInstrDesc), "r"(accumulate)
        : "memory");
}
// the mbarrier's phase completes when every MMA issued so far by this thread is done
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// 16 consecutive fp32 columns of this warp's 32 lanes (one lane per thread)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Stage outputs o0 .. o0+OT of hidden layer l: wT[k][r] = W[o0 + r][k]
// (k < win) and the per-output rows par[j][r] (bias; FiLM gamma/beta of
// this set on the first layer; sine frequencies).  A warp copies 4 weight
// rows x 8 consecutive k per instruction: 32-byte global segments, and with
// the row stride = 4 (mod 32) the 32 shared stores hit 32 banks.  Rows past
// the layer's width are left as they are (their outputs are not used).
__device__ __forceinline__ void stage_hidden_tile(const GenParams &p, int l, int o0, int set, float *wT) {
    const int win = p.widths[l];
    const int end = p.widths[l + 1];
    const float *W = p.W[l];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rr = lane >> 3, kk = lane & 7;
    for (int r0 = 4 * warp; r0 < OT; r0 += 4 * (NT / 32)) {
        const int r = r0 + rr;
        if (o0 + r >= end) continue;
        const float *src = W + (int64_t)(o0 + r) * win;
        for (int k0 = 0; k0 < win; k0 += 8) {
            const int k = k0 + kk;
            if (k < win) cpa4(wT + k * OTS + r, src + k);
        }
    }
    float *par = wT + p.ka * OTS;
    const bool film = l == 0 && p.gamma;
    for (int r = threadIdx.x; r < OT; r += NT) {
        const int o = o0 + r;
        if (o >= end) continue;
        cpa4(par + r, p.b[l] + o);
        if (film) {
            cpa4(par + OT + r, p.gamma + (int64_t)set * end + o);
            cpa4(par + 2 * OT + r, p.beta + (int64_t)set * end + o);
        }
        if (p.om[l]) cpa4(par + 3 * OT + r, p.om[l] + o);
    }
}

// acc[a][c] = sum_k act[k][4tx + a] * wT[k][CPT*ty + c], k ascending.
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
        const float4 wv = *reinterpret_cast<const float4 *>(wp + k * OTS);
        const float x[4] = {av.x, av.y, av.z, av.w};
        const float w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < CPT; ++c) acc[a][c] = fmaf(w[c], x[a], acc[a][c]);
    }
}

// Stage outputs o0 .. o0+MT of the last layer as the MMA's A operand (hi
// and lo parts; rows and K columns past the layer are zero) and their bias
// and decay rows.  A warp takes 8 rows x 4 K chunks per step: 64 contiguous
// bytes of each weight row, and each quarter-warp's 8 chunk stores fill one
// 128-byte core matrix.
__device__ __forceinline__ void stage_last_tile(const GenParams &p, int o0, int lend, float *a_hi, float *a_lo,
                                                float *lpar) {
    const int K = p.widths[p.nl - 1];
    const int kpad = p.kpad;
    const int nkc = kpad >> 2;
    const float *W = p.W[p.nl - 1];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int rr = lane & 7, kq = lane >> 3;
    const int ngroups = (MT / 8) * ((nkc + 3) >> 2);
    // batches of 4 steps: the 4 loads are in flight together before any store
    for (int it0 = warp; it0 < ngroups; it0 += 4 * (NT / 32)) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int it = it0 + u * (NT / 32);
            const int g = it % (MT / 8), j = it / (MT / 8);
            const int o = o0 + 8 * g + rr, k = 4 * (4 * j + kq);
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (it < ngroups && k < K && o < lend) {
                const float *src = W + (int64_t)o * K + k;
                if (p.vec_w) {                       // K % 4 == 0: the chunk is whole
                    v[u] = ldv4(src);
                } else {
                    v[u].x = ldv(src);
                    if (k + 1 < K) v[u].y = ldv(src + 1);
                    if (k + 2 < K) v[u].z = ldv(src + 2);
                    if (k + 3 < K) v[u].w = ldv(src + 3);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int it = it0 + u * (NT / 32);
            const int g = it % (MT / 8), j = it / (MT / 8);
            const int kc = 4 * j + kq;
            if (it < ngroups && kc < nkc) store_split(a_hi, a_lo, umma_chunk(8 * g + rr, kc, kpad), v[u]);
        }
    }
    for (int r = threadIdx.x; r < MT; r += NT) {
        const int o = o0 + r;
        lpar[r] = o < lend ? ldv(p.b[p.nl - 1] + o) : 0.f;
        lpar[MT + r] = o < lend ? ldv(p.alpha + o) * kLog2e : 0.f;   // e^{-a n} = 2^{-a log2(e) n}
    }
}

__global__ void __launch_bounds__(NT, 2) filter_gen_kernel(const GenParams p) {
    extern __shared__ __align__(1024) float sm[];
    // hidden phase: actA, actB [ka][P] and two weight buffers; last phase: the
    // A operand (hi, lo) over the same floats
    float *actA = sm;
    float *actB = actA + p.ka * P;
    float *const wbase = actB + p.ka * P;
    float *a_hi = sm;
    float *a_lo = sm + MT * p.kpad;
    float *b_hi = sm + p.u_floats;                  // B operand: the last layer's input activations
    float *b_lo = b_hi + P * p.kpad;
    float *lpar = b_lo + P * p.kpad;                // bias, alpha*log2(e) of the current tile
    __shared__ float s_norm[P];                     // window argument per position (t/L or |r|/g; squared for GAUSS)
    __shared__ int s_valid[P];
    __shared__ uint32_t s_tmem;
    __shared__ uint64_t s_bar;
    __shared__ int s_abort;

    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int64_t p0 = (int64_t)blockIdx.x * P;
    const int set = blockIdx.y;
    const int nl = p.nl;
    const int nh = nl - 1;                          // hidden layers
    const int nout = p.widths[nl];
    const int lbeg = blockIdx.z * p.out_chunk;
    const int lend = min(nout, lbeg + p.out_chunk);
    const int kpad = p.kpad;

    // accumulator columns in tensor memory (warp 0 allocates and frees them)
    if (tid < 32) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&s_tmem)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    if (tid == 0) {
        mbar_init(&s_bar, 1);
        mbar_init_fence();
        s_abort = 0;
    }

    if (nh > 0) {
        stage_hidden_tile(p, 0, 0, set, wbase);
        cpa_commit();
    }

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

    if (p.window == HY_WIN_GAUSS)
        for (int pos = tid; pos < P; pos += NT) s_norm[pos] *= s_norm[pos];

    // ---- hidden layers (a2) on the FP32 pipes; the last one writes the B operand
    if (nh > 0) {
        float *cur = actA, *nxt = actB;
        int l = 0, o0 = 0, buf = 0;
        while (l < nh) {
            // next tile in the sequence, prefetched into the other buffer
            int nl_l = l, nl_o = o0 + OT;
            if (nl_o >= p.widths[l + 1]) {
                nl_l = l + 1;
                nl_o = 0;
            }
            if (nl_l < nh) {
                stage_hidden_tile(p, nl_l, nl_o, set, wbase + (buf ^ 1) * p.wbuf);
                cpa_commit();
                cpa_wait<1>();
            } else {
                cpa_wait<0>();
            }
            __syncthreads();   // weight tile and the previous layer's activations visible

            const float *wT = wbase + buf * p.wbuf;
            const float *par = wT + p.ka * OTS;
            float acc[4][CPT];
            tile_gemm(cur, wT, p.widths[l], tx, ty, acc);
            const int wout = p.widths[l + 1];
            const bool film = (l == 0) && p.gamma;
            float v[4][CPT];   // [position][output]
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const int r = CPT * ty + c;
                const bool live = o0 + r < wout;
                const float bo = live ? par[r] : 0.f;
                const float gm = (live && film) ? par[OT + r] : 0.f;
                const float bt = (live && film) ? par[2 * OT + r] : 0.f;
                const float om = (live && p.om[l]) ? par[3 * OT + r] : 1.f;
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    float x = acc[a][c] + bo;
                    if (film) x = fmaf(1.f + gm, x, bt);
                    if (p.act == HY_ACT_SILU) x = silu(x);
                    else if (p.act == HY_ACT_SINE) x = sinf(om * x);
                    v[a][c] = live ? x : 0.f;
                }
            }
            if (l < nh - 1) {
#pragma unroll
                for (int c = 0; c < CPT; ++c) {
                    const int o = o0 + CPT * ty + c;
                    if (o < wout)
                        *reinterpret_cast<float4 *>(nxt + o * P + 4 * tx) =
                            make_float4(v[0][c], v[1][c], v[2][c], v[3][c]);
                }
            } else {
                // chunk kc = (o0 + 4 ty) / 4 holds this thread's 4 outputs for each of its 4 positions
                const int kc = (o0 >> 2) + ty;
                if (4 * kc < kpad) {
#pragma unroll
                    for (int a = 0; a < 4; ++a)
                        store_split(b_hi, b_lo, umma_chunk(4 * tx + a, kc, kpad),
                                    make_float4(v[a][0], v[a][1], v[a][2], v[a][3]));
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
    } else {
        // single-layer MLP: the encoding itself is the last layer's input
        __syncthreads();
        const int w0 = p.widths[0];
        for (int idx = tid; idx < P * (kpad >> 2); idx += NT) {
            const int pos = idx % P, kc = idx / P;
            float e[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) e[i] = (4 * kc + i < w0) ? actA[(4 * kc + i) * P + pos] : 0.f;
            store_split(b_hi, b_lo, umma_chunk(pos, kc, kpad), make_float4(e[0], e[1], e[2], e[3]));
        }
    }

    // ---- last layer on the tensor cores, 128 outputs per tile
    tc_fence_before();
    __syncthreads();   // B operand written; the hidden buffers are free for the A operand
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    const int warp = tid >> 5, lane = tid & 31;
    const int quarter = warp & 3, half = warp >> 2;   // TMEM lanes 32*quarter.., columns 32*half..
    uint32_t phase = 0;
    bool pending = false;                              // thread 0: a commit not yet seen complete
    for (int o0 = lbeg; o0 < lend; o0 += MT) {
        stage_last_tile(p, o0, lend, a_hi, a_lo, lpar);
        fence_proxy_async_smem();                      // generic writes -> tensor-core reads
        __syncthreads();
        if (tid == 0) {
            tc_fence_after();
            const uint32_t ah = smem_u32(a_hi), al = smem_u32(a_lo), bh = smem_u32(b_hi), bl = smem_u32(b_lo);
            for (int kk = 0; kk < (kpad >> 3); ++kk) {
                const uint32_t off = (uint32_t)kk * 256u;   // two 128-byte K chunks per MMA
                umma_tf32(tmem, umma_desc(al + off, kpad), umma_desc(bh + off, kpad), kk > 0);
                umma_tf32(tmem, umma_desc(ah + off, kpad), umma_desc(bl + off, kpad), 1u);
                umma_tf32(tmem, umma_desc(ah + off, kpad), umma_desc(bh + off, kpad), 1u);
            }
            umma_commit(&s_bar);
            pending = true;
        }
        if (!mbar_wait(&s_bar, phase)) {
            record_fault(p.fault, HY_FAULT_FILTER_MMA);
            s_abort = 1;
        } else if (tid == 0) {
            pending = false;
        }
        phase ^= 1;
        tc_fence_after();

        // epilogue: this thread's output row, 32 positions
        uint32_t v[32];
        uint32_t (&v0)[16] = *reinterpret_cast<uint32_t (*)[16]>(v);
        uint32_t (&v1)[16] = *reinterpret_cast<uint32_t (*)[16]>(v + 16);
        const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(32 * half);
        tmem_ld16(taddr, v0);
        tmem_ld16(taddr + 16, v1);
        tmem_wait_ld();
        const int r = 32 * quarter + lane;
        const int o = o0 + r;
        if (o < lend && !s_abort) {
            const float bo = lpar[r], al = lpar[MT + r];
            const int pb = 32 * half;
            float out[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
                out[j] = s_valid[pb + j] ? (__uint_as_float(v[j]) + bo) * exp2f(-al * s_norm[pb + j]) : 0.f;
            float *dst = p.h + ((int64_t)set * nout + o) * p.npos + p0 + pb;
            if (p.vec_out && p0 + P <= p.npos) {
#pragma unroll
                for (int j = 0; j < 32; j += 4)
                    *reinterpret_cast<float4 *>(dst + j) = make_float4(out[j], out[j + 1], out[j + 2], out[j + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (p0 + pb + j < p.npos) dst[j] = out[j];
            }
        }
        tc_fence_before();
        __syncthreads();   // accumulator read and A operand consumed before the next tile
        if (s_abort) break;
    }
    // a commit that was not seen complete may still be writing tensor memory
    if (tid == 0 && pending && !mbar_wait(&s_bar, phase ^ 1)) record_fault(p.fault, HY_FAULT_FILTER_MMA);
    __syncthreads();
    if (tid < 32) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
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
    for (int l = 0; l <= p.nl; ++l) {
        p.widths[l] = d.widths[l];
        if (l < p.nl && d.widths[l] > MAXW)
            return set_error(HY_ERR_UNSUPPORTED, "layer input width %d > %d", d.widths[l], MAXW);
    }
    // activation rows: the inputs of the hidden layers (or the encoding alone)
    p.ka = d.widths[0];
    for (int l = 1; l < p.nl - 1; ++l) p.ka = d.widths[l] > p.ka ? d.widths[l] : p.ka;
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
    const int klast = d.widths[p.nl - 1];
    p.vec_w = (klast % 4 == 0) && ((uintptr_t)d.W[p.nl - 1] % 16 == 0);
    p.kpad = (klast + 7) / 8 * 8;
    p.h = h;
    p.fault = device_fault_word();
    if (!p.fault) return set_error(HY_ERR_CUDA, "filter_gen: device fault word unavailable");
    p.wbuf = p.ka * OTS + NPAR * OT;            // a multiple of 4 floats: buffers stay 16-byte aligned
    const int64_t hidden_floats = 2LL * p.ka * P + (p.nl > 1 ? 2LL * p.wbuf : 0);
    const int64_t aop_floats = 2LL * MT * p.kpad;
    const int64_t u = hidden_floats > aop_floats ? hidden_floats : aop_floats;
    p.u_floats = (int)((u + 255) / 256 * 256);  // 1 KB aligned B operand after it
    const int64_t nblk = (p.npos + P - 1) / P;
    if (nblk > 0x7fffffffLL || d.n_sets > 65535) return set_error(HY_ERR_UNSUPPORTED, "filter grid too large");
    const size_t smem = sizeof(float) * ((size_t)p.u_floats + 2 * (size_t)P * p.kpad + 2 * (size_t)MT);
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
    const int ntile = (nout + MT - 1) / MT;
    int chunks = 1;
    if (base < (int64_t)sms) chunks = (int)((sms + base - 1) / base);
    if (chunks > ntile) chunks = ntile;
    const int per = (ntile + chunks - 1) / chunks;
    p.out_chunk = per * MT;
    chunks = (ntile + per - 1) / per;
    dim3 grid((unsigned)nblk, (unsigned)d.n_sets, (unsigned)chunks);
    filter_gen_kernel<<<grid, NT, smem, s>>>(p);
    return check_launch("filter_gen launch");
}

}  // namespace hy
