// status.h -- thread-local error message plumbing behind hyena_last_error().
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include "../../include/hyena.h"

namespace hy {

// Records a formatted message for hyena_last_error() and returns s.
hy_status set_error(hy_status s, const char *fmt, ...)
#if defined(__GNUC__)
    __attribute__((format(printf, 2, 3)))
#endif
    ;
hy_status set_cuda_error(const char *what, cudaError_t e);
// Checks cudaGetLastError() after launches.
hy_status check_launch(const char *what);
void clear_error();
// Device address of the current device's fault word: kernels whose bounded
// waits give up OR an HY_FAULT_* bit into it (hyena_device_faults reads it).
// NULL if the symbol cannot be resolved.
uint32_t *device_fault_word();

}  // namespace hy
