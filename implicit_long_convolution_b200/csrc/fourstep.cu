// fourstep.cu -- multi-pass path for sequences too long for one CTA (stub).
#include "kernels.h"
#include "status.h"

namespace hy {
// Rows are processed in chunks small enough for their intermediates to stay
// in the 126 MB L2 between passes.  Per row in flight: one complex buffer of
// M points and one fp32 stash of M samples (z_{k-1} for the skip term).
static int64_t chunk_rows(int64_t rows, int log_mc) {
    const int64_t per_row = (int64_t)12 << log_mc;
    int64_t c = ((int64_t)64 << 20) / per_row;
    if (c < 1) c = 1;
    return c < rows ? c : rows;
}
size_t long_conv_workspace(int64_t B, int64_t D, int log_mc, int) {
    if (log_mc < 15 || log_mc > 22) return 0;
    return (size_t)chunk_rows(B * D, log_mc) * ((size_t)12 << log_mc);
}
hy_status launch_long_conv(const LongConvArgs &, cudaStream_t) {
    return set_error(HY_ERR_UNSUPPORTED, "multi-pass path not built");
}
size_t long_spectrum_workspace(int64_t, int) { return 0; }
hy_status launch_long_spectrum(int64_t, int64_t, int, const float *, float2 *, void *, size_t, cudaStream_t) {
    return set_error(HY_ERR_UNSUPPORTED, "multi-pass path not built");
}
}  // namespace hy
