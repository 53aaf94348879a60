// resident.cu -- entry to the on-chip path: variant selection for the
// FFT convolution and the 1-D filter-spectrum kernels.
#include <cstdlib>
#include <cstring>

#include "resident_launch.cuh"

namespace hy {

namespace {

template <int LOG_M, bool CIRC>
hy_status launch_spectrum_t(int64_t rows, int L, const float *h, float2 *H, cudaStream_t s) {
    constexpr int LOG_P = resident_log_p(LOG_M);
    constexpr int M = 1 << LOG_M;
    constexpr int T = M >> LOG_P;
    const float2 *tw = tw_stages(LOG_M, LOG_P);
    const float2 *tws = tw_split(LOG_M);
    if (!tw || !tws) return set_error(HY_ERR_CUDA, "twiddle tables missing for M=2^%d", LOG_M);
    const size_t smem = sizeof(float2) * (size_t)spad_size(M);
    auto kernel = spectrum_rows_kernel<LOG_M, CIRC>;
    hy_status st = set_smem_limit(kernel, smem, "spectrum smem attribute");
    if (st != HY_OK) return st;
    kernel<<<(unsigned)rows, T, smem, s>>>(rows, L, h, H, tw, tws);
    return check_launch("spectrum launch");
}

}  // namespace

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

static bool aligned16(const void *q) { return ((uintptr_t)q & 15u) == 0; }

bool fft_engine_tensor() {
    const char *e = std::getenv("HYENA_FFT_ENGINE");
    return e && std::strcmp(e, "tensor") == 0;
}

hy_status launch_resident_conv(const ResidentParams &p, int log_m, hy_dtype dt, bool circular,
                               cudaStream_t s) {
    if (p.n_rows <= 0) return HY_OK;
    if (p.n_rows > 0x7fffffffLL) return set_error(HY_ERR_UNSUPPORTED, "too many rows (%lld)", (long long)p.n_rows);
    if (resident_tc_eligible(p, log_m, dt, circular) && fft_engine_tensor()) return launch_resident_tc(p, s);
    const bool chain = p.K > 1;
    // one order over whole power-of-two rows, 16-byte aligned: the persistent
    // streaming kernel (TMA bulk-copy prefetch of inputs and gate)
    const int64_t full = circular ? (int64_t)2 << log_m : (int64_t)1 << log_m;
    const int esz = dt == HY_BF16 ? 2 : 4;
    const bool fits = stream_smem_bytes(log_m, esz, circular, false) <= (size_t)227 * 1024;
    if (!chain && fits && log_m >= 6 && p.L == full && aligned16(p.u) && aligned16(p.y) &&
        (!p.gate[0] || aligned16(p.gate[0]))) {
        if (dt == HY_F32)
            return circular ? dispatch_stream<float, true>(log_m, p, s) : dispatch_stream<float, false>(log_m, p, s);
        return circular ? dispatch_stream<__nv_bfloat16, true>(log_m, p, s)
                        : dispatch_stream<__nv_bfloat16, false>(log_m, p, s);
    }
    if (dt == HY_F32) {
        if (circular) return dispatch_conv<float, true, false>(log_m, p, s);
        return chain ? dispatch_conv<float, false, true>(log_m, p, s) : dispatch_conv<float, false, false>(log_m, p, s);
    }
    if (circular) return dispatch_conv<__nv_bfloat16, true, false>(log_m, p, s);
    return chain ? dispatch_conv<__nv_bfloat16, false, true>(log_m, p, s)
                 : dispatch_conv<__nv_bfloat16, false, false>(log_m, p, s);
}

hy_status launch_spectrum_1d(int64_t rows, int L, int log_m, bool circular, const float *h, float2 *H,
                             cudaStream_t s) {
    if (rows <= 0) return HY_OK;
    if (rows > 0x7fffffffLL) return set_error(HY_ERR_UNSUPPORTED, "too many rows (%lld)", (long long)rows);
    switch (log_m) {
#define HY_CASE(LM) \
    case LM: return circular ? launch_spectrum_t<LM, true>(rows, L, h, H, s) : launch_spectrum_t<LM, false>(rows, L, h, H, s);
        HY_CASE(4) HY_CASE(5) HY_CASE(6) HY_CASE(7) HY_CASE(8) HY_CASE(9) HY_CASE(10)
        HY_CASE(11) HY_CASE(12) HY_CASE(13) HY_CASE(14)
#undef HY_CASE
        default: return set_error(HY_ERR_UNSUPPORTED, "resident transform 2^%d not built", log_m);
    }
}

}  // namespace hy
