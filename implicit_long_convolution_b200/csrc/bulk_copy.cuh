// bulk_copy.cuh -- TMA bulk copies (untiled cp.async.bulk) from global into
// shared memory, completed on an mbarrier, and the bounded wait on them.
//
// One thread arms the barrier with the byte count and issues the copy; every
// thread that reads the data waits on the barrier's phase.  A wait never
// spins without limit: it gives up after kWaitLimitNs of %globaltimer (or a
// fixed number of polls, whichever comes first), ORs a fault bit into the
// device's fault word and reports failure, so the kernel can stop at its next
// row boundary and the host sees HY_ERR_TIMEOUT from hyena_device_faults().
#pragma once
#include <stdint.h>

namespace hy {

constexpr uint64_t kWaitLimitNs = 1000000000ull;   // 1 s
constexpr uint32_t kWaitMaxPolls = 1u << 24;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Barrier with `count` arrivals per phase; call from one thread, then make it
// visible (mbar_init_fence + __syncthreads) before any use.
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Orders this thread's earlier generic-proxy shared-memory accesses (after a
// CTA barrier: the whole CTA's) before later async-proxy writes.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from
// global to shared memory; the barrier's current phase completes when the
// bytes have landed.  One thread per copy; it also performs the phase's
// single arrival.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    const uint32_t b = smem_u32(bar);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(b), "r"(bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(b)
                 : "memory");
}

// Asks for `bytes` (a multiple of 16, 16-byte aligned) of global memory to be
// brought into L2 ahead of plain loads; nothing waits for it.
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the phase of parity `parity` has completed.  Returns false if
// the limit ran out first.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t b = smem_u32(bar);
    uint64_t t0 = 0;
    for (uint32_t i = 0; i < kWaitMaxPolls; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(b), "r"(parity)
            : "memory");
        if (done) return true;
        const uint64_t now = global_ns();
        if (i == 0) t0 = now;
        else if (now - t0 > limit_ns) return false;
    }
    return false;
}

// The same bounded wait for one thread that expects a long wait (tensor-core
// work): each try_wait suspends the thread for up to kSleepHintNs or until
// the phase completes, so the waiting warp issues almost nothing.
constexpr uint32_t kSleepHintNs = 20000;
__device__ __forceinline__ bool mbar_wait_sleep(uint64_t *bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
    const uint32_t b = smem_u32(bar);
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; i < kWaitMaxPolls; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(b), "r"(parity), "r"(kSleepHintNs)
            : "memory");
        if (done) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
    return false;
}

__device__ __forceinline__ void record_fault(uint32_t *word, uint32_t bit) {
    if (word) atomicOr(word, bit);
}

}  // namespace hy
