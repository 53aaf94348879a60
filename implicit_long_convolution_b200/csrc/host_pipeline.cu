// host_pipeline.cu -- copy streams of the host-buffer entry points.
#include <mutex>

#include "host_pipeline.h"
#include "status.h"

namespace hy {

hy_status host_copy_streams(cudaStream_t &in, cudaStream_t &out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static cudaStream_t tab[kMaxDevices][2] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return set_cuda_error("host copy streams: cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return set_error(HY_ERR_UNSUPPORTED, "host copy streams: device %d", dev);
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < 2; ++i) {
        if (!tab[dev][i]) {
            e = cudaStreamCreateWithFlags(&tab[dev][i], cudaStreamNonBlocking);
            if (e != cudaSuccess) {
                tab[dev][i] = nullptr;
                return set_cuda_error("host copy streams: cudaStreamCreateWithFlags", e);
            }
        }
    }
    in = tab[dev][0];
    out = tab[dev][1];
    return HY_OK;
}

hy_status check_host_ptr(const void *p, const char *who, const char *what) {
    if (!p) return set_error(HY_ERR_INVALID_ARG, "%s: %s is null", who, what);
    cudaPointerAttributes a{};
    const cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();   // plain pageable memory on older drivers
        return HY_OK;
    }
    if (a.type == cudaMemoryTypeDevice)
        return set_error(HY_ERR_INVALID_ARG, "%s: %s is device memory; this entry point takes host buffers", who, what);
    return HY_OK;
}

}  // namespace hy
