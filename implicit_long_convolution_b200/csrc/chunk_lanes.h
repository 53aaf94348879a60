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

constexpr int kMaxLanes = 2;                 // chunk pipelines at most (streams, workspace buffers)

struct ChunkLanes {
    cudaStream_t extra[kMaxLanes - 1] = {};  // the library's streams beside the caller's
    cudaEvent_t fork = nullptr;
    cudaEvent_t join[kMaxLanes - 1] = {};
    std::mutex mu;
};
// The current device's lanes, or nullptr when the streams could not be made
// (then everything runs on the caller's stream).
ChunkLanes *chunk_lanes_of_device();

// Forks the library's streams off the caller's (holding the device's lanes
// while the call launches) or, with one lane, does nothing; chunk ci runs in
// lane lane_of(ci) on stream_of(ci), and join() puts the caller's stream
// behind the others.
struct LaneScope {
    ChunkLanes *l = nullptr;
    cudaStream_t s = nullptr;
    int n = 1;
    std::unique_lock<std::mutex> lock;
    hy_status open(int lanes, cudaStream_t caller) {
        s = caller;
        n = 1;
        if (lanes < 2) return HY_OK;
        l = chunk_lanes_of_device();
        if (!l) return HY_OK;                  // no second stream: one lane
        lock = std::unique_lock<std::mutex>(l->mu);
        n = lanes < kMaxLanes ? lanes : kMaxLanes;
        cudaError_t e = cudaEventRecord(l->fork, caller);
        for (int i = 0; i + 1 < n && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(l->extra[i], l->fork, 0);
        if (e != cudaSuccess) {
            lock.unlock();
            l = nullptr;
            n = 1;
            return set_cuda_error("chunk stream fork", e);
        }
        return HY_OK;
    }
    int lanes() const { return n; }
    int lane_of(int ci) const { return n > 1 ? ci % n : 0; }
    cudaStream_t stream_of(int ci) const {
        const int ln = lane_of(ci);
        return ln == 0 ? s : l->extra[ln - 1];
    }
    hy_status join() {
        if (!l) return HY_OK;
        cudaError_t e = cudaSuccess;
        for (int i = 0; i + 1 < n; ++i) {
            cudaError_t e1 = cudaEventRecord(l->join[i], l->extra[i]);
            if (e1 == cudaSuccess) e1 = cudaStreamWaitEvent(s, l->join[i], 0);
            if (e == cudaSuccess) e = e1;
        }
        lock.unlock();
        l = nullptr;
        n = 1;
        return e == cudaSuccess ? HY_OK : set_cuda_error("chunk stream join", e);
    }
    ~LaneScope() { join(); }
};

// Lanes for `units` work units in chunks of `per_chunk` units of
// `unit_bytes` each, given `ws_bytes` of workspace: one per chunk buffer the
// workspace holds, at most one per chunk and at most kMaxLanes.
inline int chunk_lanes(int64_t units, int64_t per_chunk, size_t unit_bytes, size_t ws_bytes) {
    const size_t chunk_bytes = (size_t)per_chunk * unit_bytes;
    const int64_t chunks = (units + per_chunk - 1) / per_chunk;
    int64_t n = chunk_bytes ? (int64_t)(ws_bytes / chunk_bytes) : 1;
    if (n > chunks) n = chunks;
    if (n > kMaxLanes) n = kMaxLanes;
    return n < 1 ? 1 : (int)n;
}
// Recommended workspace: one chunk buffer per lane that can be busy.
inline size_t chunk_workspace(int64_t units, int64_t per_chunk, size_t unit_bytes) {
    const int64_t chunks = (units + per_chunk - 1) / per_chunk;
    const int64_t n = chunks < kMaxLanes ? chunks : kMaxLanes;
    return (size_t)(n < 1 ? 1 : n) * (size_t)per_chunk * unit_bytes;
}

}  // namespace hy
