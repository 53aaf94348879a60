// chunk_lanes.h -- two chunk pipelines for the chunked multi-pass paths
// (the long-sequence four-step passes and the 3-D transform passes).
//
// With more than one chunk and a workspace of two chunk buffers,
// consecutive chunks alternate between the caller's stream and a second
// stream of the library's (one per device, created on first use and kept),
// each chunk in its own buffer: the passes of one chunk then run in the
// tail waves of the other's instead of after them (the passes are
// latency-bound; a chunk's last wave leaves most SMs idle).  The second
// stream joins the caller's by events, so the call stays ordered on the
// caller's stream and can be captured into a graph.  Calls from several host
// threads on one device take turns on the second stream.
#pragma once
#include <cuda_runtime.h>
#include <mutex>

#include "status.h"

namespace hy {

constexpr int kMaxLanes = 2;

struct ChunkLanes {
    cudaStream_t s2 = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex mu;
};
// The current device's lanes, or nullptr when the second stream could not be
// made (then everything runs on the caller's stream).
ChunkLanes *chunk_lanes_of_device();

// Forks the second stream off the caller's (holding the device's lanes while
// the call launches) or, with one lane, does nothing; stream_of(ci) names
// chunk ci's stream, and join() puts the caller's stream behind the second.
struct LaneScope {
    ChunkLanes *l = nullptr;
    cudaStream_t s = nullptr;
    std::unique_lock<std::mutex> lock;
    hy_status open(int lanes, cudaStream_t caller) {
        s = caller;
        if (lanes < 2) return HY_OK;
        l = chunk_lanes_of_device();
        if (!l) return HY_OK;                  // no second stream: one lane
        lock = std::unique_lock<std::mutex>(l->mu);
        cudaError_t e = cudaEventRecord(l->fork, caller);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(l->s2, l->fork, 0);
        if (e != cudaSuccess) {
            lock.unlock();
            l = nullptr;
            return set_cuda_error("chunk stream fork", e);
        }
        return HY_OK;
    }
    int lanes() const { return l ? 2 : 1; }
    cudaStream_t stream_of(int ci) const { return (l && (ci & 1)) ? l->s2 : s; }
    hy_status join() {
        if (!l) return HY_OK;
        cudaError_t e = cudaEventRecord(l->join, l->s2);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, l->join, 0);
        lock.unlock();
        l = nullptr;
        return e == cudaSuccess ? HY_OK : set_cuda_error("chunk stream join", e);
    }
    ~LaneScope() { join(); }
};

// Lanes for `units` work units in chunks of `per_chunk` units of
// `unit_bytes` each, given `ws_bytes` of workspace.
inline int chunk_lanes(int64_t units, int64_t per_chunk, size_t unit_bytes, size_t ws_bytes) {
    const size_t chunk_bytes = (size_t)per_chunk * unit_bytes;
    return (units > per_chunk && ws_bytes >= (size_t)kMaxLanes * chunk_bytes) ? kMaxLanes : 1;
}

}  // namespace hy
