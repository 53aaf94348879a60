// resident_stream_f32.cu -- fp32-I/O streaming variants of the on-chip path.
#include "resident_launch.cuh"
namespace hy {
template hy_status dispatch_stream<float, false>(int, const ResidentParams &, cudaStream_t);
template hy_status dispatch_stream<float, true>(int, const ResidentParams &, cudaStream_t);
}  // namespace hy
