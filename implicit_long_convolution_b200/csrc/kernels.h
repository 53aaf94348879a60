// kernels.h -- internal launcher declarations (host side).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hyena.h"

namespace hy {

struct ResidentParams;

hy_status launch_resident_conv(const ResidentParams &p, int log_m, hy_dtype dt, bool circular,
                               cudaStream_t s);
// one order over bf16 rows of L = 8192 with the radix-32 FFT stages on the
// tensor cores (resident_tc.cu)
bool resident_tc_eligible(const ResidentParams &p, int log_m, hy_dtype dt, bool circular);
hy_status launch_resident_tc(ResidentParams p, cudaStream_t s);
// FFT engine for the transforms that have a tensor-core version: the fp32
// SIMT kernel (faster, see the measurements) unless the environment
// variable HYENA_FFT_ENGINE is "tensor" (read at every call, so both can be
// run and compared in one process).
bool fft_engine_tensor();
int device_sm_count();

// Fused backward of the order-2 operator (bw_fused.cu): L a power of two in
// [512, 8192] whose shared-memory plan fits, the ptrs16 16-byte aligned.
bool bw_fused_eligible(int order, int L, hy_dtype dt, const void *const *ptrs16, int nptrs);
hy_status launch_bw_fused(int B, int D, int L, hy_dtype dt, const void *v, const void *x1, const void *dy,
                          const void *H, const float *Dsk, void *dv, void *dx1, float *dh, float *dD,
                          cudaStream_t s);

// 2-D TMA tensor map over `outer` rows of `inner` elements (row pitch
// row_bytes), box box_inner x box_outer, reads past the extent land as zeros
// (tma_map.cu).  The map covers this GPU's memory only.
hy_status tma_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                     const char *who);
hy_status launch_spectrum_1d(int64_t rows, int L, int log_m, bool circular, const float *h, float2 *H,
                             cudaStream_t s);

// filter generator (filter_gen.cu); desc validated by the caller
hy_status launch_filter_gen(const hy_filter_desc &d, float *h, cudaStream_t s);

// multi-pass (four-step) path for long sequences (fourstep.cu)
struct LongConvArgs {
    int K;                         // orders
    int64_t B, D, L;               // rows are (B, D), length L
    int log_mc;                    // complex transform length M = 2^log_mc (n = 2M)
    hy_dtype dt;
    const void *u;
    const void *gate[8];
    const float2 *spec[8];         // (D, M+1) per order
    const float *skip[8];
    void *y;
    void *ws;
    size_t ws_bytes;
};
// Workspace of the multi-pass path: the recommended size (two chunk buffers
// when there is more than one chunk: the chunks then alternate between two
// streams) and the minimum (one chunk buffer: one stream).
size_t long_conv_workspace(int64_t B, int64_t D, int log_mc, int K);
size_t long_conv_workspace_min(int64_t B, int64_t D, int log_mc);
hy_status launch_long_conv(const LongConvArgs &a, cudaStream_t s);
size_t long_spectrum_workspace(int64_t rows, int log_mc);
size_t long_spectrum_workspace_min(int64_t rows, int log_mc);
hy_status launch_long_spectrum(int64_t rows, int64_t L, int log_mc, const float *h, float2 *H, void *ws,
                               size_t ws_bytes, cudaStream_t s);

// Multi-pass operator with its workspace in a static device array
// (fourstep.cu); no allocation by anyone.
size_t noalloc_scratch_bytes();
hy_status launch_long_conv_noalloc(const LongConvArgs &a, cudaStream_t s);

// backward-pass element-wise and reduction kernels (backward.cu)
hy_status bw_to_f32(const void *src, hy_dtype dt, float *dst, int64_t n, cudaStream_t s);
hy_status bw_from_f32(const float *src, hy_dtype dt, void *dst, int64_t n, cudaStream_t s);
hy_status bw_gate(const void *x, hy_dtype dt, const float *c, float *z, int64_t n, cudaStream_t s);
hy_status bw_dx_e(const float *g, const float *c, const void *x, hy_dtype dt, void *dx, float *er, int64_t rows, int L,
                  cudaStream_t s);
hy_status bw_next_g(const float *r, float *g, const void *x, hy_dtype dt, const float *Dk, int64_t rows, int D, int L,
                    cudaStream_t s);
hy_status bw_dh(const float *w, float *dh, int B, int D, int L, cudaStream_t s);
hy_status bw_dD(const float *g, const void *x, hy_dtype dt, const float *z, float *dD, int B, int D, int L,
                cudaStream_t s);

// streaming decode of the spectral gate with a prefix-FFT cache (decode.cu)
struct GateDecodeArgs {
    int64_t rows;                  // B * H * Dh
    int n;                         // transform length (power of two)
    int64_t pos;                   // position of the new token, 0 <= pos < n
    int64_t dh, heads;             // gate row of row r: (r / dh) % heads, sample r / (dh * heads)
    const float2 *g;
    int64_t g_batch_stride;        // complex elements; 0 = shared
    float2 *cache;                 // rows x (n/2 + 1), updated in place
};
hy_status launch_gate_decode(const GateDecodeArgs &a, hy_dtype dt, const void *x, const void *x2, void *y,
                             cudaStream_t s);

// N-D path (ndconv.cu)
struct NDArgs {
    int g[3];                      // grid
    int S[3];                      // transform grid
    int circular;
    int64_t B, D;
    const float *u;
    const float2 *H;
    int64_t H_batch_stride;
    const float *skip;
    const float *gate;
    float *y;
    void *ws;
    size_t ws_bytes;
};
// Workspace of the 3-D passes: the recommended size (two chunk buffers when
// there is more than one chunk) or, with `minimum`, one chunk buffer.
size_t nd_conv_workspace(const int g[3], int circular, int64_t B, int64_t D, bool minimum = false);
hy_status launch_nd_conv(const NDArgs &a, cudaStream_t s);
size_t nd_spectrum_workspace(int64_t rows, const int S[3], bool minimum = false);
hy_status launch_nd_spectrum(int64_t rows, const int S[3], const float *h, float2 *H, void *ws,
                             size_t ws_bytes, cudaStream_t s);

}  // namespace hy
