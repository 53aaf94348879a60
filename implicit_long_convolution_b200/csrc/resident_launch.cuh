// resident_launch.cuh -- launch templates of the on-chip path; each
// dispatch_conv<IO, CIRC, CHAIN> is instantiated in its own .cu file so the
// heavy kernel variants compile in parallel.
#pragma once
#include "kernels.h"
#include "resident.cuh"
#include "status.h"
#include "twiddle.h"

namespace hy {

template <typename Kern>
inline hy_status set_smem_limit(Kern kernel, size_t smem, const char *what) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return set_cuda_error(what, e);
    }
    return HY_OK;
}

template <int LOG_M, typename IO, bool CIRC, bool CHAIN>
hy_status launch_conv_t(ResidentParams p, cudaStream_t s) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int T = M >> LOG_P;
    p.tw_fft = tw_stages(LOG_M, LOG_P);
    p.tw_split = tw_split(LOG_M);
    if (!p.tw_fft || !p.tw_split) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^%d", LOG_M);
    const size_t smem = sizeof(float2) * (size_t)spad_size(M);
    auto kernel = resident_conv_kernel<LOG_M, IO, CIRC, CHAIN>;
    hy_status st = set_smem_limit(kernel, smem, "resident conv smem attribute");
    if (st != HY_OK) return st;
    kernel<<<(unsigned)p.n_rows, T, smem, s>>>(p);
    return check_launch("resident conv launch");
}

template <typename IO, bool CIRC, bool CHAIN>
hy_status dispatch_conv(int log_m, const ResidentParams &p, cudaStream_t s) {
    switch (log_m) {
#define HY_CASE(LM) \
    case LM: return launch_conv_t<LM, IO, CIRC, CHAIN>(p, s);
        HY_CASE(4) HY_CASE(5) HY_CASE(6) HY_CASE(7) HY_CASE(8) HY_CASE(9) HY_CASE(10)
        HY_CASE(11) HY_CASE(12) HY_CASE(13) HY_CASE(14)
#undef HY_CASE
        default: return set_error(HY_ERR_UNSUPPORTED, "resident transform 2^%d not built", log_m);
    }
}

// ---- streaming (persistent, TMA bulk-copy prefetch) variant
int device_sm_count();

template <int LOG_M, typename IO, bool CIRC>
hy_status launch_stream_t(ResidentParams p, cudaStream_t s) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int T = M >> LOG_P;
    constexpr bool PF = stream_pf_gate(LOG_M, (int)sizeof(IO), CIRC);
    p.tw_fft = tw_stages(LOG_M, LOG_P);
    p.tw_split = tw_split(LOG_M);
    if (!p.tw_fft || !p.tw_split) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^%d", LOG_M);
    p.fault = device_fault_word();
    if (!p.fault) return set_error(HY_ERR_CUDA, "device fault word unavailable");
    const size_t smem = stream_smem_bytes(LOG_M, (int)sizeof(IO), CIRC, PF);
    auto kernel = resident_stream_kernel<LOG_M, IO, CIRC, PF>;
    hy_status st = set_smem_limit(kernel, smem, "stream conv smem attribute");
    if (st != HY_OK) return st;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, T, smem);
    if (e != cudaSuccess) return set_cuda_error("occupancy query", e);
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)per_sm * device_sm_count();
    if (grid > p.n_rows) grid = p.n_rows;
    kernel<<<(unsigned)grid, T, smem, s>>>(p);
    return check_launch("stream conv launch");
}

template <typename IO, bool CIRC>
hy_status dispatch_stream(int log_m, const ResidentParams &p, cudaStream_t s) {
    switch (log_m) {
#define HY_CASE(LM) \
    case LM: return launch_stream_t<LM, IO, CIRC>(p, s);
        HY_CASE(6) HY_CASE(7) HY_CASE(8) HY_CASE(9) HY_CASE(10)
        HY_CASE(11) HY_CASE(12) HY_CASE(13) HY_CASE(14)
#undef HY_CASE
        default: return set_error(HY_ERR_UNSUPPORTED, "stream transform 2^%d not built", log_m);
    }
}

extern template hy_status dispatch_stream<float, false>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_stream<float, true>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_stream<__nv_bfloat16, false>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_stream<__nv_bfloat16, true>(int, const ResidentParams &, cudaStream_t);

extern template hy_status dispatch_conv<float, false, false>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_conv<float, false, true>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_conv<__nv_bfloat16, false, false>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_conv<__nv_bfloat16, false, true>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_conv<float, true, false>(int, const ResidentParams &, cudaStream_t);
extern template hy_status dispatch_conv<__nv_bfloat16, true, false>(int, const ResidentParams &, cudaStream_t);

}  // namespace hy
