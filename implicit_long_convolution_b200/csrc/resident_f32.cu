// resident_f32.cu -- fp32-I/O causal variants of the on-chip path.
#include "resident_launch.cuh"
namespace hy {
template hy_status dispatch_conv<float, false, false>(int, const ResidentParams &, cudaStream_t);
template hy_status dispatch_conv<float, false, true>(int, const ResidentParams &, cudaStream_t);
}  // namespace hy
