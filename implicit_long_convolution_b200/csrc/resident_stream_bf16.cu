// resident_stream_bf16.cu -- bf16-I/O streaming variants of the on-chip path.
#include "resident_launch.cuh"
namespace hy {
template hy_status dispatch_stream<__nv_bfloat16, false>(int, const ResidentParams &, cudaStream_t);
template hy_status dispatch_stream<__nv_bfloat16, true>(int, const ResidentParams &, cudaStream_t);
}  // namespace hy
