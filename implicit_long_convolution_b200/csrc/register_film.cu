// register_film.cu -- input conditioning of the HyenaND kernel ([ND]
// 방법론: HyenaND, 레지스터 및 FiLM을 통한 입력 의존적 커널): R register tokens are
// processed with each input sample; the control variable z(x) is the
// softmax-weighted mean of their activations, and z(x) modulates the
// kernel's coordinate MLP through FiLM.
//
//   l[b, r]  = query · reg[b, r] (query given) + scores[b, r] (scores given)
//   w[b, :]  = softmax(l[b, :])            (maximum subtracted)
//   z[b, :]  = Σ_r w[b, r] reg[b, r, :]
//   (gamma[b], beta[b]) = W z[b] + bias    (W: (2H, C); gamma = first H rows)
//
// gamma / beta are the film_gamma / film_beta of hyena_filter_gen (FiLM of
// the first hidden layer: (1 + gamma) ⊙ y + beta).  One CTA per sample: the
// logits by warp-strided dot products, the softmax in one warp, z in shared
// memory, then one warp per FiLM output.  fp32 arithmetic throughout.
#include "common.cuh"
#include "status.h"

namespace hy {

namespace {

constexpr int NT = 256;
constexpr int MAX_R = 1024;
constexpr int MAX_C = 8192;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__global__ void __launch_bounds__(NT) register_film_kernel(int R, int C, int H, const float *__restrict__ reg,
                                                           const float *__restrict__ query,
                                                           const float *__restrict__ scores,
                                                           const float *__restrict__ W,
                                                           const float *__restrict__ bias, float *__restrict__ gamma,
                                                           float *__restrict__ beta) {
    extern __shared__ float sm[];
    float *z = sm;              // [C]
    float *w = sm + C;          // [R]
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = NT / 32;
    const float *rb = reg + (int64_t)b * R * C;

    // logits, one warp per register
    for (int r = warp; r < R; r += nw) {
        float acc = 0.f;
        if (query) {
            const float *row = rb + (int64_t)r * C;
            for (int c = lane; c < C; c += 32) acc = fmaf(__ldg(query + c), __ldg(row + c), acc);
            acc = warp_sum(acc);
        }
        if (lane == 0) w[r] = acc + (scores ? __ldg(scores + (int64_t)b * R + r) : 0.f);
    }
    __syncthreads();
    // softmax over the R logits (warp 0)
    if (warp == 0) {
        float m = -INFINITY;
        for (int r = lane; r < R; r += 32) m = fmaxf(m, w[r]);
        m = warp_max(m);
        float s = 0.f;
        for (int r = lane; r < R; r += 32) {
            const float e = expf(w[r] - m);
            w[r] = e;
            s += e;
        }
        s = warp_sum(s);
        const float inv = 1.f / s;
        for (int r = lane; r < R; r += 32) w[r] *= inv;
    }
    __syncthreads();
    // z = Σ_r w[r] reg[r, :]
    for (int c = threadIdx.x; c < C; c += NT) {
        float acc = 0.f;
        for (int r = 0; r < R; ++r) acc = fmaf(w[r], __ldg(rb + (int64_t)r * C + c), acc);
        z[c] = acc;
    }
    __syncthreads();
    // FiLM parameters: one warp per output row of W
    for (int o = warp; o < 2 * H; o += nw) {
        const float *wr = W + (int64_t)o * C;
        float acc = 0.f;
        for (int c = lane; c < C; c += 32) acc = fmaf(__ldg(wr + c), z[c], acc);
        acc = warp_sum(acc);
        if (lane == 0) {
            const float v = acc + (bias ? __ldg(bias + o) : 0.f);
            if (o < H) gamma[(int64_t)b * H + o] = v;
            else beta[(int64_t)b * H + (o - H)] = v;
        }
    }
}

}  // namespace

}  // namespace hy

using namespace hy;

extern "C" hy_status hyena_register_film(int B, int R, int C, int H, const float *reg, const float *query,
                                         const float *scores, const float *W_film, const float *b_film,
                                         float *gamma, float *beta, void *stream) {
    clear_error();
    const char *who = "hyena_register_film";
    if (B < 1 || R < 1 || C < 1 || H < 1)
        return set_error(HY_ERR_INVALID_ARG, "%s: B, R, C, H must be >= 1", who);
    if (R > MAX_R || C > MAX_C)
        return set_error(HY_ERR_UNSUPPORTED, "%s: R <= %d and C <= %d", who, MAX_R, MAX_C);
    if (!reg || !W_film || !gamma || !beta) return set_error(HY_ERR_INVALID_ARG, "%s: null pointer", who);
    if (gamma == beta) return set_error(HY_ERR_INVALID_ARG, "%s: gamma and beta alias", who);
    const size_t smem = sizeof(float) * ((size_t)C + (size_t)R);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(register_film_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)smem);
        if (e != cudaSuccess) return set_cuda_error("hyena_register_film: shared memory attribute", e);
    }
    register_film_kernel<<<(unsigned)B, NT, smem, (cudaStream_t)stream>>>(R, C, H, reg, query, scores, W_film, b_film,
                                                                         gamma, beta);
    return check_launch("hyena_register_film");
}
