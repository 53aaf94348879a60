// filter_gen.cu -- fused implicit filter generator.
//
// [HN] 아키텍처 상세, step 2: h(t) = FFN(pos_enc(t)) · w(t), w(t) = e^{-αt};
// [ES] 어떻게 동작하나요?: a small MLP with sinusoidal features and an
// exponential decay window; [ND] 방법론: HyenaND: coordinate MLP on the N-D
// grid with FiLM conditioning per sample.
//
// One CTA evaluates TP = 64 positions of one filter set for one chunk of the
// outputs of the last layer (grid z; only as many chunks as fill the GPU): it builds the positional
// encoding in shared memory, runs every MLP layer as a small fp32 GEMM
// (register tile of 4 positions x 4 outputs per thread, weights staged in
// shared memory 64 outputs at a time), applies FiLM and SiLU on hidden
// layers and the decay window on the last one, and writes the filter rows
// with the position index fastest (coalesced).  The hidden layers are
// recomputed per output chunk; they are a small part of the work when the
// last layer is wide, and the chunks give the grid enough CTAs.
#include "kernels.h"
#include "status.h"

namespace hy {

namespace {

constexpr int TP = 64;          // positions per CTA
constexpr int NT = 256;         // threads
constexpr int OC = 64;          // outputs per weight chunk
constexpr int WS = OC + 4;      // row stride of the staged (transposed) weights (float4-aligned)
constexpr int MAXW = 132;       // max layer width (input encoding or hidden), multiple of 4
constexpr int MAXL = 4;

struct GenParams {
    int ndim;
    int64_t L;                  // 1-D length
    int g, S, circular;         // 3-D
    int F, include_t;
    int nl;
    int widths[MAXL + 1];
    const float *W[MAXL];
    const float *b[MAXL];
    int act;
    const float *gamma, *beta;
    const float *alpha;
    int64_t npos;               // positions per set (L or S^3)
    int out_chunk;              // last-layer outputs per CTA (grid z), multiple of OC
    float *h;
};

__device__ __forceinline__ float silu(float a) { return a / (1.f + expf(-a)); }

__device__ __forceinline__ int signed_off(int i, int S) { return i < S / 2 ? i : i - S; }

__global__ void __launch_bounds__(NT) filter_gen_kernel(const GenParams p) {
    extern __shared__ float sm[];
    float *actA = sm;                      // [MAXW][TP]
    float *actB = actA + MAXW * TP;        // [MAXW][TP]
    float *wt = actB + MAXW * TP;          // [MAXW][WS] transposed weight chunk
    __shared__ float s_norm[TP];           // decay argument per position (t/L or |r|/g)
    __shared__ int s_valid[TP];

    const int tid = threadIdx.x;
    const int64_t p0 = (int64_t)blockIdx.x * TP;
    const int set = blockIdx.y;

    // ---- positional encoding (a1) into actA[feature][pos]
    const int w0 = p.widths[0];
    for (int pos = tid; pos < TP; pos += NT) {
        const int64_t q = p0 + pos;
        s_valid[pos] = q < p.npos;
        s_norm[pos] = 0.f;
    }
    if (p.ndim == 1) {
        for (int idx = tid; idx < TP * w0; idx += NT) {
            const int pos = idx % TP, f = idx / TP;
            const int64_t tt = p0 + pos;
            float v = 0.f;
            if (tt < p.npos) {
                if (p.include_t && f == 0) {
                    v = (float)((double)tt / (double)p.L);
                } else {
                    const int ff = f - p.include_t;      // 0..2F-1
                    const int j = (ff % p.F) + 1;
                    const int64_t r = ((int64_t)j * tt) % p.L;
                    float s, c;
                    sincospif((float)(2.0 * (double)r / (double)p.L), &s, &c);
                    v = (ff < p.F) ? c : s;
                }
            }
            actA[f * TP + pos] = v;
        }
        for (int pos = tid; pos < TP; pos += NT) {
            const int64_t tt = p0 + pos;
            s_norm[pos] = (float)((double)tt / (double)p.L);
        }
    } else {
        const int S = p.S;
        for (int idx = tid; idx < TP * w0; idx += NT) {
            const int pos = idx % TP, f = idx / TP;
            const int64_t q = p0 + pos;
            float v = 0.f;
            if (q < p.npos) {
                const int axis = f / (2 * p.F);
                const int ff = f % (2 * p.F);
                const int j = (ff % p.F) + 1;
                const int ia = axis == 0 ? (int)(q / ((int64_t)S * S)) : (axis == 1 ? (int)((q / S) % S) : (int)(q % S));
                const int ra = signed_off(ia, S);
                const int twog = 2 * p.g;
                int mm = (j * ra) % twog;
                if (mm < 0) mm += twog;
                float s, c;
                sincospif((float)mm / (float)p.g, &s, &c);     // angle π j r / g
                v = (ff < p.F) ? c : s;
            }
            actA[f * TP + pos] = v;
        }
        for (int pos = tid; pos < TP; pos += NT) {
            const int64_t q = p0 + pos;
            if (q < p.npos) {
                const int r0 = signed_off((int)(q / ((int64_t)S * S)), S);
                const int r1 = signed_off((int)((q / S) % S), S);
                const int r2 = signed_off((int)(q % S), S);
                bool inside = true;
                if (!p.circular) inside = (abs(r0) < p.g) && (abs(r1) < p.g) && (abs(r2) < p.g);
                s_valid[pos] = inside ? 1 : 0;
                s_norm[pos] = sqrtf((float)(r0 * r0 + r1 * r1 + r2 * r2)) / (float)p.g;
            }
        }
    }
    __syncthreads();

    // ---- MLP layers (a2)
    const int tx = tid % (TP / 4), ty = tid / (TP / 4);   // positions tx*4.., outputs ty*4..
    float *cur = actA, *nxt = actB;
    for (int l = 0; l < p.nl; ++l) {
        const int win = p.widths[l], wout = p.widths[l + 1];
        const bool last = (l == p.nl - 1);
        const float *W = p.W[l];
        const float *bias = p.b[l];
        const int obeg = last ? blockIdx.z * p.out_chunk : 0;
        const int oend = last ? min(wout, obeg + p.out_chunk) : wout;
        for (int o0 = obeg; o0 < oend; o0 += OC) {
            // stage W[o0 .. o0+OC)[0..win) transposed (row stride OC+4 keeps
            // the float4 reads aligned): consecutive threads read consecutive
            // inputs of one output row (coalesced)
            {
                const int lane = tid & 31, wid = tid >> 5;
                for (int oo = wid; oo < OC; oo += NT / 32) {
                    const bool ok = o0 + oo < oend;
                    const float *wrow = W + (int64_t)(o0 + oo) * win;
                    for (int i = lane; i < win; i += 32) wt[i * WS + oo] = ok ? __ldg(wrow + i) : 0.f;
                }
            }
            __syncthreads();
            float acc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
            for (int i = 0; i < win; ++i) {
                const float4 av = *reinterpret_cast<const float4 *>(cur + i * TP + tx * 4);
                const float4 wv = *reinterpret_cast<const float4 *>(wt + i * WS + ty * 4);
                const float aa[4] = {av.x, av.y, av.z, av.w};
                const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(ww[c], aa[a], acc[a][c]);
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int o = o0 + ty * 4 + c;
                if (o >= oend) continue;
                const float bo = __ldg(bias + o);
                if (!last) {
                    float gm = 0.f, bt = 0.f;
                    const bool film = (l == 0) && p.gamma;
                    if (film) {
                        gm = __ldg(p.gamma + (int64_t)set * wout + o);
                        bt = __ldg(p.beta + (int64_t)set * wout + o);
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        float v = acc[a][c] + bo;
                        if (film) v = fmaf(1.f + gm, v, bt);
                        if (p.act == HY_ACT_SILU) v = silu(v);
                        nxt[o * TP + tx * 4 + a] = v;
                    }
                } else {
                    // last layer: decay window, staged in the free activation
                    // buffer as [output][position] for coalesced row stores
                    const float al = __ldg(p.alpha + o);
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const int pos = tx * 4 + a;
                        float v = (acc[a][c] + bo) * expf(-al * s_norm[pos]);
                        if (!s_valid[pos]) v = 0.f;
                        nxt[(o - o0) * TP + pos] = v;
                    }
                }
            }
            __syncthreads();
            if (last) {
                const int nrow = min(OC, oend - o0);
                for (int idx = tid; idx < nrow * TP; idx += NT) {
                    const int ol = idx / TP, pos = idx % TP;
                    if (p0 + pos < p.npos) p.h[((int64_t)set * wout + o0 + ol) * p.npos + p0 + pos] = nxt[ol * TP + pos];
                }
                __syncthreads();
            }
        }
        float *tmp = cur;
        cur = nxt;
        nxt = tmp;
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
    p.F = d.n_freq;
    p.include_t = d.include_t;
    p.nl = d.n_layers;
    if (p.nl < 1 || p.nl > MAXL) return set_error(HY_ERR_UNSUPPORTED, "n_layers must be 1..%d", MAXL);
    for (int l = 0; l <= p.nl; ++l) {
        p.widths[l] = d.widths[l];
        if (l < p.nl && d.widths[l] > MAXW)
            return set_error(HY_ERR_UNSUPPORTED, "layer input width %d > %d", d.widths[l], MAXW);
    }
    for (int l = 0; l < p.nl; ++l) {
        p.W[l] = d.W[l];
        p.b[l] = d.b[l];
    }
    p.act = d.act;
    p.gamma = d.film_gamma;
    p.beta = d.film_beta;
    p.alpha = d.alpha;
    p.npos = d.ndim == 1 ? (int64_t)d.L : (int64_t)p.S * p.S * p.S;
    p.h = h;
    const int64_t nblk = (p.npos + TP - 1) / TP;
    if (nblk > 0x7fffffffLL || d.n_sets > 65535) return set_error(HY_ERR_UNSUPPORTED, "filter grid too large");
    const size_t smem = sizeof(float) * (size_t)(2 * MAXW * TP + MAXW * WS);
    cudaError_t e = cudaFuncSetAttribute(filter_gen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return set_cuda_error("filter_gen smem attribute", e);
    // split the last layer over grid z only as far as needed to fill the GPU
    // (each split recomputes the hidden layers)
    const int nout = d.widths[d.n_layers];
    const int64_t base = nblk * d.n_sets;
    int sms = 148;
    {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    }
    const int max_chunks = (nout + OC - 1) / OC;
    int chunks = (int)((2 * (int64_t)sms + base - 1) / base);
    if (chunks < 1) chunks = 1;
    if (chunks > max_chunks) chunks = max_chunks;
    p.out_chunk = ((nout + chunks - 1) / chunks + OC - 1) / OC * OC;
    chunks = (nout + p.out_chunk - 1) / p.out_chunk;
    dim3 grid((unsigned)nblk, (unsigned)d.n_sets, (unsigned)chunks);
    filter_gen_kernel<<<grid, NT, smem, s>>>(p);
    return check_launch("filter_gen launch");
}

}  // namespace hy
