// host_pipeline.h -- host-buffer entry points: copy in, compute, copy out,
// overlapped chunk by chunk.
//
// The rows of a call are cut into chunks.  Chunk c uses slot c mod 3 of a
// device ring carved from the caller's workspace.  Its inputs are copied on a
// copy-in stream, it is computed on the caller's stream, and its output is
// copied back on a copy-out stream.  Events order the three, so the
// host-to-device copy of chunk c+1, the compute of chunk c and the
// device-to-host copy of chunk c-1 run at the same time (PCIe is full
// duplex).  The call only enqueues work; the caller's stream waits for the
// last copy-out, so synchronising that stream makes the host output valid.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hyena.h"
#include "status.h"

namespace hy {

constexpr int kHostSlots = 3;                       // device ring slots
constexpr size_t kHostChunkBytes = (size_t)16 << 20;  // target bytes of one input per chunk

// The two copy streams of the current device (created once, non-blocking).
hy_status host_copy_streams(cudaStream_t &in, cudaStream_t &out);

// Host pointer check: rejects device memory (managed and host memory pass).
hy_status check_host_ptr(const void *p, const char *who, const char *what);

inline size_t round256(size_t b) { return (b + 255) & ~(size_t)255; }

// One chunk: n_in inputs of in_bytes each (host sources), one output of
// out_bytes (host destination).
struct HostChunk {
    const void *src[9];
    size_t in_bytes;
    void *dst;
    size_t out_bytes;
};

// Runs `nchunks` chunks.  describe(c, chunk) fills chunk c; compute(c,
// dev_in, dev_out, stream) enqueues its work on `stream` reading dev_in[i]
// and writing dev_out.  slot_in / slot_out: per-slot capacity of one input
// and of the output (bytes); ring: device memory of
// kHostSlots * (n_in * round256(slot_in) + round256(slot_out)) bytes.
template <class Describe, class Compute>
hy_status run_host_pipeline(int n_in, int nchunks, size_t slot_in, size_t slot_out, char *ring,
                            cudaStream_t stream, Describe describe, Compute compute, const char *who) {
    cudaStream_t s_in, s_out;
    hy_status st = host_copy_streams(s_in, s_out);
    if (st != HY_OK) return st;
    const size_t in_stride = round256(slot_in);
    const size_t slot_bytes = (size_t)n_in * in_stride + round256(slot_out);
    cudaEvent_t ev_entry = nullptr, ev_in[kHostSlots] = {}, ev_comp[kHostSlots] = {}, ev_out[kHostSlots] = {};
    auto release = [&]() {
        // pending events are released by the runtime once they complete
        if (ev_entry) cudaEventDestroy(ev_entry);
        for (int s = 0; s < kHostSlots; ++s) {
            if (ev_in[s]) cudaEventDestroy(ev_in[s]);
            if (ev_comp[s]) cudaEventDestroy(ev_comp[s]);
            if (ev_out[s]) cudaEventDestroy(ev_out[s]);
        }
    };
    cudaError_t e = cudaEventCreateWithFlags(&ev_entry, cudaEventDisableTiming);
    for (int s = 0; s < kHostSlots && e == cudaSuccess; ++s) {
        e = cudaEventCreateWithFlags(&ev_in[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_comp[s], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_out[s], cudaEventDisableTiming);
    }
    // the copy streams start after everything already queued on the caller's
    // stream (earlier users of the ring, producers of the spectra)
    if (e == cudaSuccess) e = cudaEventRecord(ev_entry, stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_entry, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_entry, 0);
    if (e != cudaSuccess) {
        release();
        return set_cuda_error(who, e);
    }
    for (int c = 0; c < nchunks; ++c) {
        const int s = c % kHostSlots;
        HostChunk ch{};
        describe(c, ch);
        char *slot = ring + (size_t)s * slot_bytes;
        const void *dev_in[9];
        for (int i = 0; i < n_in; ++i) dev_in[i] = slot + (size_t)i * in_stride;
        void *dev_out = slot + (size_t)n_in * in_stride;
        // copy in once the slot's previous chunk has been computed
        if (c >= kHostSlots) e = cudaStreamWaitEvent(s_in, ev_comp[s], 0);
        for (int i = 0; i < n_in && e == cudaSuccess; ++i)
            e = cudaMemcpyAsync(const_cast<void *>(dev_in[i]), ch.src[i], ch.in_bytes, cudaMemcpyHostToDevice, s_in);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in[s], s_in);
        // compute once the inputs are in and the slot's previous output is out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ev_in[s], 0);
        if (e == cudaSuccess && c >= kHostSlots) e = cudaStreamWaitEvent(stream, ev_out[s], 0);
        if (e != cudaSuccess) {
            release();
            return set_cuda_error(who, e);
        }
        st = compute(c, dev_in, dev_out, stream);
        if (st != HY_OK) {
            release();
            return st;
        }
        e = cudaEventRecord(ev_comp[s], stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_comp[s], 0);
        if (e == cudaSuccess) e = cudaMemcpyAsync(ch.dst, dev_out, ch.out_bytes, cudaMemcpyDeviceToHost, s_out);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out[s], s_out);
        if (e != cudaSuccess) {
            release();
            return set_cuda_error(who, e);
        }
    }
    // the caller's stream continues after the last copy-out
    for (int s = 0; s < kHostSlots && s < nchunks && e == cudaSuccess; ++s) e = cudaStreamWaitEvent(stream, ev_out[s], 0);
    release();
    if (e != cudaSuccess) return set_cuda_error(who, e);
    return HY_OK;
}

}  // namespace hy
