// faults.cu -- the device fault word behind hyena_device_faults() and the
// self-test of the bounded wait.
//
// Kernels never trap and never spin without limit: a bounded wait that gives
// up ORs an HY_FAULT_* bit into one word per device (a static __device__
// variable, so no allocation) and the kernel returns early.  The host reads
// the word on a stream of its choice, after the work it wants checked.
#include <mutex>

#include "bulk_copy.cuh"
#include "status.h"

namespace hy {

namespace {

__device__ uint32_t g_fault_word;

std::mutex g_mu;
uint32_t *g_word[64] = {nullptr};

// One CTA arms an mbarrier that expects two arrivals, makes one, and waits on
// the phase with the given limit: the phase cannot complete, so the wait runs
// out, records HY_FAULT_SELFTEST and the kernel returns.
__global__ void selftest_wait_kernel(uint32_t *word, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        mbar_init_fence();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
        if (!mbar_wait(&bar, 0, limit_ns)) record_fault(word, HY_FAULT_SELFTEST);
    }
}

}  // namespace

uint32_t *device_fault_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_word[dev]) {
        void *a = nullptr;
        if (cudaGetSymbolAddress(&a, g_fault_word) != cudaSuccess) return nullptr;
        g_word[dev] = static_cast<uint32_t *>(a);
    }
    return g_word[dev];
}

}  // namespace hy

extern "C" hy_status hyena_device_faults(uint32_t *faults, int clear, void *stream) {
    using namespace hy;
    clear_error();
    if (!faults) return set_error(HY_ERR_INVALID_ARG, "hyena_device_faults: null output");
    *faults = 0;
    uint32_t *word = device_fault_word();
    if (!word) return set_error(HY_ERR_CUDA, "hyena_device_faults: fault word unavailable");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, word, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return set_cuda_error("hyena_device_faults: read", e);
    if (clear && v) {
        e = cudaMemsetAsync(word, 0, sizeof(uint32_t), s);
        if (e != cudaSuccess) return set_cuda_error("hyena_device_faults: clear", e);
    }
    *faults = v;
    if (v) return set_error(HY_ERR_TIMEOUT, "a bounded device wait gave up (fault bits 0x%x)", v);
    return HY_OK;
}

extern "C" hy_status hyena_selftest_bounded_wait(uint32_t limit_us, void *stream) {
    using namespace hy;
    clear_error();
    if (limit_us == 0 || limit_us > 1000000u)
        return set_error(HY_ERR_INVALID_ARG, "hyena_selftest_bounded_wait: limit must be 1..1000000 us");
    uint32_t *word = device_fault_word();
    if (!word) return set_error(HY_ERR_CUDA, "hyena_selftest_bounded_wait: fault word unavailable");
    selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(word, (uint64_t)limit_us * 1000ull);
    return check_launch("selftest launch");
}
