// projection.cu -- input projection of the operator ([HN] 아키텍처 상세, step 1:
// v, x_1, ..., x_{N-1} = split(W_proj · x), a learnable linear map of the
// token activations), written straight into the channel-major (B, D, L)
// layout the convolution reads, with the bias added in the epilogue.
//
//   out_k[b, d, l] = bias[k D + d] + Σ_c W[k D + d, c] · x[b, l, c]
//
// For sample b this is the GEMM  Out[m, l] = Σ_c W[m, c] · x[b, l, c]  with
// m = k D + d.  Both operands are K-major as they sit in memory (c is the
// contiguous index of W's rows and of x's tokens), and row m of the result is
// the contiguous row (b, d) of out_k -- so the transpose into the
// channel-major layout is free: one thread of the epilogue owns one row m of
// the tile and writes its sequence positions as 16-byte runs.
//
// bf16: a persistent, warp-specialised tcgen05 kernel, one CTA per SM.
//   warp 0    TMA producer: 128 x 64 tiles of W and 256 x 64 tiles of x
//             (128-byte swizzle) into a 4-stage shared-memory ring;
//   warp 1    allocates 512 TMEM columns (two 128 x 256 fp32 accumulators)
//             and issues the MMAs (M = 128, N = 256, K = 16, bf16 x bf16 ->
//             fp32) from one thread; each stage is released to the
//             producer by tcgen05.commit, each finished tile handed to the
//             epilogue the same way;
//   warps 2-5 epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//             output row per thread), + bias in fp32, one rounding to bf16,
//             vector stores; the other accumulator is being filled
//             meanwhile.
// Tiles run n-major (consecutive tiles share the x tile, W stays in L2).
// Every wait is bounded: one that gives up records HY_FAULT_PROJECTION in the
// device fault word and the CTA winds down (the producer waits for the
// copies it issued, the MMA thread for its MMAs) before freeing TMEM.
//
// fp32: plain fp32 FMA arithmetic (no TF32), a tiled SIMT kernel with the
// same fused bias and channel-major stores.
#include <cuda.h>
#include <cuda_bf16.h>
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "status.h"
#include "tcgen05.cuh"

namespace hy {

namespace {

constexpr int MAX_OUT = 9;

// ---------------------------------------------------------------- bf16: tcgen05
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t A_BYTES = BM * BK * 2;           // 16 KB
constexpr uint32_t B_BYTES = BN * BK * 2;           // 32 KB
constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t ACC_COLS = BN;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int NT_TC = 192;
constexpr size_t TC_SMEM = (size_t)STAGES * STAGE_BYTES + 1024;   // + 1024-byte alignment slack
constexpr uint32_t IDESC = tc::idesc_f16(BM, BN, true);

struct ProjParams {
    int M, L, C, D;
    int tiles_m, tiles_l;       // tiles along m, along l per sample
    int64_t n_tiles;
    const float *bias;
    void *out[MAX_OUT];
    uint32_t *fault;
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__global__ void __launch_bounds__(NT_TC, 1)
proj_tc_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX, const ProjParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
    __shared__ uint32_t s_tmem;
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 1) tc::tmem_alloc(&s_tmem, TMEM_COLS);
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);             // one arrival per epilogue warp
        }
        mbar_init(&drain, 1);
        mbar_init_fence();
        s_abort = 0;
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s_tmem;
    const int nk = (p.C + BK - 1) / BK;
    auto give_up = [&]() {
        record_fault(p.fault, HY_FAULT_PROJECTION);
        s_abort = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, armed_ph = 0;      // per stage: a load was issued, and its phase parity
            for (int64_t t = blockIdx.x; t < p.n_tiles && !s_abort; t += gridDim.x) {
                const int mt = (int)(t % p.tiles_m);
                const int64_t nt = t / p.tiles_m;
                const int b = (int)(nt / p.tiles_l);
                const int l0 = (int)(nt % p.tiles_l) * BN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1)) {
                        give_up();
                        break;
                    }
                    uint8_t *sa = smem + (size_t)s * STAGE_BYTES;
                    tc::mbar_expect_tx(&full[s], STAGE_BYTES);
                    tc::tma_load_2d(sa, &tmW, kb * BK, mt * BM, &full[s]);
                    tc::tma_load_2d(sa + A_BYTES, &tmX, kb * BK, b * p.L + l0, &full[s]);
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
            }
            // no copy may still be landing when the CTA exits
            for (int q = 0; q < STAGES; ++q)
                if ((armed >> q) & 1)
                    if (!mbar_wait(&full[q], (armed_ph >> q) & 1)) record_fault(p.fault, HY_FAULT_PROJECTION);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.n_tiles && ok && !s_abort; t += gridDim.x) {
                if (!mbar_wait(&tempty[acc], aph ^ 1)) {
                    give_up();
                    break;
                }
                tc::fence_after();
                const uint32_t d = tmem + (uint32_t)acc * ACC_COLS;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!mbar_wait(&full[s], ph)) {
                        give_up();
                        ok = false;
                        break;
                    }
                    tc::fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * STAGE_BYTES);
                    const uint64_t ad = tc::desc_k_sw128(sa), bd = tc::desc_k_sw128(sa + A_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)     // K step of 16 elements = 32 bytes = 2 descriptor units
                        tc::mma_f16(d, ad + 2 * k, bd + 2 * k, IDESC, (kb | k) != 0);
                    tc::commit(&empty[s]);                // the stage is free once these MMAs have read it
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1;
                    }
                }
                if (!ok) break;
                tc::commit(&tfull[acc]);                  // the tile's accumulator is complete
                if (++acc == 2) {
                    acc = 0;
                    aph ^= 1;
                }
            }
            // every MMA issued has finished before TMEM is freed
            tc::commit(&drain);
            if (!mbar_wait(&drain, 0)) record_fault(p.fault, HY_FAULT_PROJECTION);
        }
    } else {
        // ---- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31
        const int q = warp & 3;
        const int row = q * 32 + lane;
        int acc = 0;
        uint32_t aph = 0;
        for (int64_t t = blockIdx.x; t < p.n_tiles && !s_abort; t += gridDim.x) {
            // the warp takes one decision (tcgen05.ld below is warp-wide)
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[acc], aph))) {
                give_up();
                break;
            }
            tc::fence_after();
            const int mt = (int)(t % p.tiles_m);
            const int64_t nt = t / p.tiles_m;
            const int b = (int)(nt / p.tiles_l);
            const int l0 = (int)(nt % p.tiles_l) * BN;
            const int m = mt * BM + row;
            const bool valid = m < p.M;
            const int ko = valid ? m / p.D : 0;
            const int dd = valid ? m % p.D : 0;
            const float bias = (valid && p.bias) ? __ldg(p.bias + m) : 0.f;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(p.out[ko]) + ((int64_t)b * p.D + dd) * p.L;
            const bool vec = (p.L & 7) == 0;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + (uint32_t)acc * ACC_COLS + (uint32_t)(c * 32) + ((uint32_t)(q * 32) << 16), v);
                tc::tmem_wait_ld();
                if (!valid) continue;
                const int l = l0 + c * 32;
                if (vec && l + 32 <= p.L) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + l);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(v[8 * j + 0]) + bias, __uint_as_float(v[8 * j + 1]) + bias);
                        w.y = pack_bf16(__uint_as_float(v[8 * j + 2]) + bias, __uint_as_float(v[8 * j + 3]) + bias);
                        w.z = pack_bf16(__uint_as_float(v[8 * j + 4]) + bias, __uint_as_float(v[8 * j + 5]) + bias);
                        w.w = pack_bf16(__uint_as_float(v[8 * j + 6]) + bias, __uint_as_float(v[8 * j + 7]) + bias);
                        dst[j] = w;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (l + j < p.L) orow[l + j] = __float2bfloat16_rn(__uint_as_float(v[j]) + bias);
                }
            }
            tc::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
            if (++acc == 2) {
                acc = 0;
                aph ^= 1;
            }
        }
    }
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    __syncwarp();
    if (warp == 1) tc::tmem_free(tmem, TMEM_COLS);
}

// ---------------------------------------------------------------- fp32: SIMT
constexpr int FM = 128, FN = 128, FK = 16, NT_F = 256;

__global__ void __launch_bounds__(NT_F) proj_f32_kernel(const float *__restrict__ x, const float *__restrict__ W,
                                                        const ProjParams p, int B) {
    __shared__ float As[FK][FM + 4];     // As[k][m] = W[m0 + m, k0 + k]
    __shared__ float Bs[FK][FN + 4];     // Bs[k][l] = x[b, l0 + l, k0 + k]
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.x * FM;
    const int l0 = blockIdx.y * FN;
    const int b = blockIdx.z;
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    const float *xb = x + (int64_t)b * p.L * p.C;
    for (int k0 = 0; k0 < p.C; k0 += FK) {
        // 128 rows x 16 k of each operand: 8 elements per thread, k fastest
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = tid + e * NT_F;
            const int r = idx >> 4, k = idx & 15;
            const int gm = m0 + r, gl = l0 + r, gk = k0 + k;
            As[k][r] = (gm < p.M && gk < p.C) ? __ldg(W + (int64_t)gm * p.C + gk) : 0.f;
            Bs[k][r] = (gl < p.L && gk < p.C) ? __ldg(xb + (int64_t)gl * p.C + gk) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < FK; ++k) {
            float a[8], bv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = As[k][ty * 8 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                bv[j] = Bs[k][tx * 4 + j];
                bv[4 + j] = Bs[k][64 + tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + ty * 8 + i;
        if (m >= p.M) continue;
        const float bias = p.bias ? __ldg(p.bias + m) : 0.f;
        float *orow = reinterpret_cast<float *>(p.out[m / p.D]) + ((int64_t)b * p.D + m % p.D) * p.L;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int l = l0 + h * 64 + tx * 4;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (l + j < p.L) orow[l + j] = acc[i][4 * h + j] + bias;
        }
    }
}

// ---------------------------------------------------------------- host side
std::mutex g_mu;
bool g_attr_set[64] = {};

hy_status launch_tc(int B, int L, int C, int D, int n_out, const void *x, const void *W, const float *bias,
                    void *const *out, cudaStream_t s) {
    const int M = n_out * D;
    // W and x as 2-D bf16 arrays (rows of C elements), boxes of 64 x 128 and
    // 64 x 256 with the 128-byte swizzle; reads past the extent land as zeros
    CUtensorMap mw, mx;
    hy_status st = tma_map_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, (uint64_t)C, (uint64_t)M, (uint64_t)C * 2, BK,
                              BM, CU_TENSOR_MAP_SWIZZLE_128B, "hyena_projection");
    if (st != HY_OK) return st;
    st = tma_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, (uint64_t)C, (uint64_t)B * L, (uint64_t)C * 2, BK, BN,
                    CU_TENSOR_MAP_SWIZZLE_128B, "hyena_projection");
    if (st != HY_OK) return st;
    ProjParams p{};
    p.M = M;
    p.L = L;
    p.C = C;
    p.D = D;
    p.tiles_m = (M + BM - 1) / BM;
    p.tiles_l = (L + BN - 1) / BN;
    p.n_tiles = (int64_t)p.tiles_m * p.tiles_l * B;
    p.bias = bias;
    for (int k = 0; k < n_out; ++k) p.out[k] = out[k];
    p.fault = device_fault_word();
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (dev >= 0 && dev < 64 && !g_attr_set[dev]) {
            const cudaError_t e =
                cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TC_SMEM);
            if (e != cudaSuccess) return set_cuda_error("hyena_projection: shared memory attribute", e);
            g_attr_set[dev] = true;
        }
    }
    const int64_t grid = p.n_tiles < sms ? p.n_tiles : sms;
    proj_tc_kernel<<<(unsigned)grid, NT_TC, TC_SMEM, s>>>(mw, mx, p);
    return check_launch("hyena_projection (tcgen05 GEMM)");
}

hy_status launch_f32(int B, int L, int C, int D, int n_out, const float *x, const float *W, const float *bias,
                     void *const *out, cudaStream_t s) {
    ProjParams p{};
    p.M = n_out * D;
    p.L = L;
    p.C = C;
    p.D = D;
    p.bias = bias;
    for (int k = 0; k < n_out; ++k) p.out[k] = out[k];
    if (B > 65535) return set_error(HY_ERR_UNSUPPORTED, "hyena_projection: fp32 path takes B <= 65535");
    dim3 grid((unsigned)((p.M + FM - 1) / FM), (unsigned)((L + FN - 1) / FN), (unsigned)B);
    proj_f32_kernel<<<grid, NT_F, 0, s>>>(x, W, p, B);
    return check_launch("hyena_projection (fp32 GEMM)");
}

}  // namespace

}  // namespace hy

using namespace hy;

extern "C" size_t hyena_projection_workspace(void) { return 0; }

extern "C" hy_status hyena_projection(int B, int L, int C, int D, int n_out, hy_dtype dt, const void *x,
                                      const void *W, const float *bias, void *const *out, void *ws,
                                      size_t ws_bytes, void *stream) {
    (void)ws;
    (void)ws_bytes;
    clear_error();
    const char *who = "hyena_projection";
    if (B < 1 || L < 1 || C < 1 || D < 1 || n_out < 1 || n_out > MAX_OUT)
        return set_error(HY_ERR_INVALID_ARG, "%s: B, L, C, D must be >= 1 and n_out in 1..9", who);
    if (dt != HY_F32 && dt != HY_BF16) return set_error(HY_ERR_INVALID_ARG, "%s: unknown dtype", who);
    if (!x || !W || !out) return set_error(HY_ERR_INVALID_ARG, "%s: null pointer", who);
    for (int k = 0; k < n_out; ++k)
        if (!out[k]) return set_error(HY_ERR_INVALID_ARG, "%s: out[%d] is null", who, k);
    const size_t esz = dt == HY_BF16 ? 2 : 4;
    if ((uintptr_t)x % 16 || (uintptr_t)W % 16 || (C * esz) % 16)
        return set_error(HY_ERR_INVALID_ARG, "%s: x and W must be 16-byte aligned with rows of a multiple of 16 bytes", who);
    for (int k = 0; k < n_out; ++k)
        if ((uintptr_t)out[k] % 16) return set_error(HY_ERR_INVALID_ARG, "%s: out[%d] misaligned", who, k);
    if ((int64_t)n_out * D > (int64_t)1 << 30 || (int64_t)B * L > ((int64_t)1 << 31) - 1)
        return set_error(HY_ERR_UNSUPPORTED, "%s: n_out*D and B*L must stay below 2^30 and 2^31", who);
    if (dt == HY_BF16) return launch_tc(B, L, C, D, n_out, x, W, bias, out, (cudaStream_t)stream);
    return launch_f32(B, L, C, D, n_out, reinterpret_cast<const float *>(x), reinterpret_cast<const float *>(W), bias,
                      out, (cudaStream_t)stream);
}
