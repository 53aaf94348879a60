// resident_circ.cu -- circular (spectral gate) variants of the on-chip path.
#include "resident_launch.cuh"
namespace hy {
template hy_status dispatch_conv<float, true, false>(int, const ResidentParams &, cudaStream_t);
template hy_status dispatch_conv<__nv_bfloat16, true, false>(int, const ResidentParams &, cudaStream_t);
}  // namespace hy
