// status.cu -- thread-local last-error message.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "status.h"

namespace hy {

static thread_local char g_msg[512] = "";

hy_status set_error(hy_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
    va_end(ap);
    return s;
}

hy_status set_cuda_error(const char *what, cudaError_t e) {
    return set_error(HY_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

hy_status check_launch(const char *what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_cuda_error(what, e);
    return HY_OK;
}

void clear_error() { g_msg[0] = 0; }

}  // namespace hy

extern "C" const char *hyena_last_error(void) { return hy::g_msg; }
