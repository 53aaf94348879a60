// projection.cu -- input projection of the operator ([HN] 아키텍처 상세, step 1:
// v, x_1, ..., x_{N-1} = split(W_proj · x), a learnable linear map of the
// token activations), written straight into the channel-major (B, D, L)
// layout the convolution reads.
//
// out_k[b, d, l] = bias[k D + d] + Σ_c W[k D + d, c] · x[b, l, c]
//
// Per output k this is one batched GEMM.  In column-major terms the output of
// sample b is the L x D matrix with leading dimension L, so
//   out_k[b] (L x D) = x[b]^T (L x C, i.e. the row-major (L, C) block read
//   transposed) · W_k^T (C x D, the row-major (D, C) block read as is)
// and the transposed layout costs nothing.  The GEMM is cuBLASLt's (bf16
// tensor cores with fp32 accumulation, or plain fp32 without TF32); the
// library is loaded on first use, so entry points that do not project never
// need it.  The bias is added by a streaming pass over the output (cuBLASLt
// offers its bias epilogue only along the other dimension of this layout).
#include <dlfcn.h>
#include <mutex>

#include <cublasLt.h>
#include <cuda_bf16.h>

#include "status.h"

namespace hy {

namespace {

struct LtApi {
    bool loaded = false;
    decltype(&cublasLtCreate) create = nullptr;
    decltype(&cublasLtMatmulDescCreate) desc_create = nullptr;
    decltype(&cublasLtMatmulDescDestroy) desc_destroy = nullptr;
    decltype(&cublasLtMatmulDescSetAttribute) desc_set = nullptr;
    decltype(&cublasLtMatrixLayoutCreate) layout_create = nullptr;
    decltype(&cublasLtMatrixLayoutDestroy) layout_destroy = nullptr;
    decltype(&cublasLtMatrixLayoutSetAttribute) layout_set = nullptr;
    decltype(&cublasLtMatmulPreferenceCreate) pref_create = nullptr;
    decltype(&cublasLtMatmulPreferenceDestroy) pref_destroy = nullptr;
    decltype(&cublasLtMatmulPreferenceSetAttribute) pref_set = nullptr;
    decltype(&cublasLtMatmulAlgoGetHeuristic) heuristic = nullptr;
    decltype(&cublasLtMatmul) matmul = nullptr;
};

std::mutex g_lt_mu;
LtApi g_lt;
cublasLtHandle_t g_lt_handle[64] = {};

hy_status load_lt() {
    if (g_lt.loaded) return HY_OK;
    void *h = dlopen("libcublasLt.so.12", RTLD_NOW | RTLD_GLOBAL);
    if (!h) h = dlopen("libcublasLt.so", RTLD_NOW | RTLD_GLOBAL);
    if (!h) return set_error(HY_ERR_UNSUPPORTED, "hyena_projection: cannot load libcublasLt (%s)", dlerror());
#define HY_SYM(field, name)                                                                              \
    g_lt.field = reinterpret_cast<decltype(g_lt.field)>(dlsym(h, #name));                               \
    if (!g_lt.field) return set_error(HY_ERR_UNSUPPORTED, "hyena_projection: libcublasLt lacks " #name);
    HY_SYM(create, cublasLtCreate)
    HY_SYM(desc_create, cublasLtMatmulDescCreate)
    HY_SYM(desc_destroy, cublasLtMatmulDescDestroy)
    HY_SYM(desc_set, cublasLtMatmulDescSetAttribute)
    HY_SYM(layout_create, cublasLtMatrixLayoutCreate)
    HY_SYM(layout_destroy, cublasLtMatrixLayoutDestroy)
    HY_SYM(layout_set, cublasLtMatrixLayoutSetAttribute)
    HY_SYM(pref_create, cublasLtMatmulPreferenceCreate)
    HY_SYM(pref_destroy, cublasLtMatmulPreferenceDestroy)
    HY_SYM(pref_set, cublasLtMatmulPreferenceSetAttribute)
    HY_SYM(heuristic, cublasLtMatmulAlgoGetHeuristic)
    HY_SYM(matmul, cublasLtMatmul)
#undef HY_SYM
    g_lt.loaded = true;
    return HY_OK;
}

hy_status lt_handle(cublasLtHandle_t &out) {
    std::lock_guard<std::mutex> lock(g_lt_mu);
    hy_status st = load_lt();
    if (st != HY_OK) return st;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("hyena_projection: cudaGetDevice", e);
    if (dev < 0 || dev >= 64) return set_error(HY_ERR_UNSUPPORTED, "hyena_projection: device %d", dev);
    if (!g_lt_handle[dev]) {
        const cublasStatus_t s = g_lt.create(&g_lt_handle[dev]);
        if (s != CUBLAS_STATUS_SUCCESS) {
            g_lt_handle[dev] = nullptr;
            return set_error(HY_ERR_CUDA, "hyena_projection: cublasLtCreate failed (%d)", (int)s);
        }
    }
    out = g_lt_handle[dev];
    return HY_OK;
}

// out[row, l] += bias[row % D] over rows = B * D rows of length L (row-major).
// Streaming pass: with L a multiple of 8 every 16-byte chunk (8 bf16 or 4
// fp32) lies in one row; each thread keeps UNROLL chunks in flight.
template <typename T>
__global__ void __launch_bounds__(256) add_bias_vec_kernel(T *out, const float *__restrict__ bias, int64_t chunks,
                                                           int D, int L) {
    constexpr int PER = 16 / sizeof(T);         // elements per chunk
    constexpr int UNROLL = 4;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t c0 = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c0 < chunks; c0 += stride * UNROLL) {
        uint4 v[UNROLL];
        float b[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t c = c0 + u * stride;
            if (c < chunks) {
                v[u] = *reinterpret_cast<const uint4 *>(out + c * PER);
                b[u] = __ldg(bias + ((c * PER) / L) % D);
            }
        }
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) {
            const int64_t c = c0 + u * stride;
            if (c >= chunks) continue;
            if constexpr (sizeof(T) == 4) {
                float4 f = *reinterpret_cast<float4 *>(&v[u]);
                f.x += b[u]; f.y += b[u]; f.z += b[u]; f.w += b[u];
                *reinterpret_cast<float4 *>(out + c * PER) = f;
            } else {
                __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v[u]);
#pragma unroll
                for (int q = 0; q < 4; ++q) h[q] = __floats2bfloat162_rn(__low2float(h[q]) + b[u], __high2float(h[q]) + b[u]);
                *reinterpret_cast<uint4 *>(out + c * PER) = v[u];
            }
        }
    }
}

// any L: one element per thread and row
template <typename T>
__global__ void __launch_bounds__(256) add_bias_kernel(T *out, const float *__restrict__ bias, int64_t rows,
                                                       int D, int L) {
    const int64_t row = blockIdx.y * (int64_t)gridDim.z + blockIdx.z;
    if (row >= rows) return;
    const float b = __ldg(bias + row % D);
    T *p = out + row * (int64_t)L;
    for (int l = blockIdx.x * blockDim.x + threadIdx.x; l < L; l += gridDim.x * blockDim.x) {
        if constexpr (sizeof(T) == 4) p[l] = p[l] + b;
        else p[l] = __float2bfloat16_rn(__bfloat162float(p[l]) + b);
    }
}

template <typename T>
hy_status add_bias(T *out, const float *bias, int64_t rows, int D, int L, cudaStream_t s) {
    if (L % 8 == 0) {
        const int64_t chunks = rows * L / (16 / sizeof(T));
        int sms = 148, dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        int64_t blocks = (chunks + 256 * 4 - 1) / (256 * 4);
        if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
        add_bias_vec_kernel<T><<<(unsigned)blocks, 256, 0, s>>>(out, bias, chunks, D, L);
    } else {
        dim3 grid((unsigned)((L + 255) / 256 < 8 ? (L + 255) / 256 : 8), (unsigned)((rows + 65534) / 65535),
                  (unsigned)(rows < 65535 ? rows : 65535));
        add_bias_kernel<T><<<grid, 256, 0, s>>>(out, bias, rows, D, L);
    }
    return check_launch("hyena_projection bias");
}

// One batched GEMM per projection k: out_k[b] as the column-major L x D
// matrix (ld L) = x[b] (stored C x L, read transposed) · W_k (stored C x D).
hy_status project_gemm(cublasLtHandle_t lt, int B, int L, int C, int D, int n_out, hy_dtype dt, const void *x,
                       const void *W, void *const *out, void *ws, cudaStream_t stream) {
    const char *who = "hyena_projection";
    const size_t esz = dt == HY_BF16 ? 2 : 4;
    const cudaDataType_t ty = dt == HY_BF16 ? CUDA_R_16BF : CUDA_R_32F;
    cublasLtMatmulDesc_t op = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, ld = nullptr;
    cublasLtMatmulPreference_t pref = nullptr;
    auto cleanup = [&]() {
        if (pref) g_lt.pref_destroy(pref);
        if (la) g_lt.layout_destroy(la);
        if (lb) g_lt.layout_destroy(lb);
        if (ld) g_lt.layout_destroy(ld);
        if (op) g_lt.desc_destroy(op);
    };
    auto fail = [&](const char *what, cublasStatus_t s) {
        cleanup();
        return set_error(HY_ERR_CUDA, "%s: %s failed (%d)", who, what, (int)s);
    };
    cublasStatus_t s = g_lt.desc_create(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F);   // no TF32: plain fp32 or bf16 MMA
    if (s != CUBLAS_STATUS_SUCCESS) return fail("cublasLtMatmulDescCreate", s);
    const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
    g_lt.desc_set(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta));
    g_lt.desc_set(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb));
    if ((s = g_lt.layout_create(&la, ty, C, L, C)) != CUBLAS_STATUS_SUCCESS) return fail("layout A", s);
    if ((s = g_lt.layout_create(&lb, ty, C, D, C)) != CUBLAS_STATUS_SUCCESS) return fail("layout B", s);
    if ((s = g_lt.layout_create(&ld, ty, L, D, L)) != CUBLAS_STATUS_SUCCESS) return fail("layout D", s);
    const int32_t batch = B;
    const int64_t sa = (int64_t)L * C, sb = 0, sd = (int64_t)L * D;   // the weights are shared by the samples
    g_lt.layout_set(la, CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &batch, sizeof(batch));
    g_lt.layout_set(la, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &sa, sizeof(sa));
    g_lt.layout_set(lb, CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &batch, sizeof(batch));
    g_lt.layout_set(lb, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &sb, sizeof(sb));
    g_lt.layout_set(ld, CUBLASLT_MATRIX_LAYOUT_BATCH_COUNT, &batch, sizeof(batch));
    g_lt.layout_set(ld, CUBLASLT_MATRIX_LAYOUT_STRIDED_BATCH_OFFSET, &sd, sizeof(sd));
    if ((s = g_lt.pref_create(&pref)) != CUBLAS_STATUS_SUCCESS) return fail("preference", s);
    const size_t wsb = (size_t)32 << 20;
    g_lt.pref_set(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &wsb, sizeof(wsb));
    cublasLtMatmulHeuristicResult_t heur{};
    int found = 0;
    s = g_lt.heuristic(lt, op, la, lb, ld, ld, pref, 1, &heur, &found);
    if (s != CUBLAS_STATUS_SUCCESS || found < 1) {
        cleanup();
        return set_error(HY_ERR_UNSUPPORTED, "%s: no cuBLASLt algorithm for this shape (%d)", who, (int)s);
    }
    const float one = 1.f, zero = 0.f;
    for (int k = 0; k < n_out; ++k) {
        const char *Wk = reinterpret_cast<const char *>(W) + (size_t)k * D * C * esz;
        s = g_lt.matmul(lt, op, &one, x, la, Wk, lb, &zero, out[k], ld, out[k], ld, &heur.algo, ws, wsb, stream);
        if (s != CUBLAS_STATUS_SUCCESS) return fail("cublasLtMatmul", s);
    }
    cleanup();
    return HY_OK;
}

}  // namespace

}  // namespace hy

using namespace hy;

extern "C" size_t hyena_projection_workspace(void) { return (size_t)32 << 20; }

extern "C" hy_status hyena_projection(int B, int L, int C, int D, int n_out, hy_dtype dt, const void *x,
                                      const void *W, const float *bias, void *const *out, void *ws,
                                      size_t ws_bytes, void *stream) {
    clear_error();
    const char *who = "hyena_projection";
    if (B < 1 || L < 1 || C < 1 || D < 1 || n_out < 1 || n_out > 9)
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
    if (!ws || ws_bytes < hyena_projection_workspace() || (uintptr_t)ws % 256)
        return set_error(HY_ERR_WORKSPACE, "%s: needs %zu bytes of 256-byte aligned workspace", who,
                         hyena_projection_workspace());
    cublasLtHandle_t lt;
    hy_status st = lt_handle(lt);
    if (st != HY_OK) return st;
    st = project_gemm(lt, B, L, C, D, n_out, dt, x, W, out, ws, (cudaStream_t)stream);
    if (st != HY_OK) return st;
    if (bias) {
        const int64_t rows = (int64_t)B * D;
        for (int k = 0; k < n_out; ++k) {
            st = dt == HY_BF16
                     ? add_bias(reinterpret_cast<__nv_bfloat16 *>(out[k]), bias + (size_t)k * D, rows, D, L,
                                (cudaStream_t)stream)
                     : add_bias(reinterpret_cast<float *>(out[k]), bias + (size_t)k * D, rows, D, L,
                                (cudaStream_t)stream);
            if (st != HY_OK) return st;
        }
    }
    return HY_OK;
}
