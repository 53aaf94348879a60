// resident_bf16.cu -- bf16-I/O causal variants of the on-chip path.
#include "resident_launch.cuh"
namespace hy {
template hy_status dispatch_conv<__nv_bfloat16, false, false>(int, const ResidentParams &, cudaStream_t);
template hy_status dispatch_conv<__nv_bfloat16, false, true>(int, const ResidentParams &, cudaStream_t);
}  // namespace hy
