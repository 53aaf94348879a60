// ndconv.cu -- N-D path (stub).
#include "kernels.h"
#include "status.h"

namespace hy {
size_t nd_conv_workspace(const int *, int, int64_t, int64_t) { return 0; }
hy_status launch_nd_conv(const NDArgs &, cudaStream_t) {
    return set_error(HY_ERR_UNSUPPORTED, "N-D path not built");
}
size_t nd_spectrum_workspace(int64_t, const int *) { return 0; }
hy_status launch_nd_spectrum(int64_t, const int *, const float *, float2 *, void *, size_t, cudaStream_t) {
    return set_error(HY_ERR_UNSUPPORTED, "N-D path not built");
}
}  // namespace hy
