// twiddle.h -- constant twiddle tables shared by the kernels.
//
// All tables are computed once on the host in double precision (angles
// reduced exactly in integers before cos/sin), rounded to fp32 and copied
// into one static __device__ array per device on first use.  No device
// memory is allocated for them.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include "../../include/hyena.h"

namespace hy {

// Stage tables of a size-2^log_m block FFT with per-thread 2^log_p elements
// (layout of fft_core.cuh: stage s at plan_tw_offset, entry (r-1)*p + k).
const float2 *tw_stages(int log_m, int log_p);
// W_{2M}^k = exp(-2πi k / 2M) for k = 0..M/2 (M = 2^log_m): the real-FFT
// split twiddles.
const float2 *tw_split(int log_m);
// W_N^j for j < 2^lo (N = 2^log_n) followed by W_N^{j * 2^lo} for j < N/2^lo:
// two-level table for W_N^e, e < N (e = hi*2^lo + lo).
const float2 *tw_pow2(int log_n, int lo_bits);

// Uploads the tables to the current device if not done yet.
hy_status tw_ensure_device();

}  // namespace hy
