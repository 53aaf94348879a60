// tma_map.cu -- host side of the TMA tensor maps: cuTensorMapEncodeTiled
// from the driver, looked up once through the runtime (the library does not
// link the driver library itself).  The maps only ever describe this GPU's
// own memory, and every load through them fills one CTA's shared memory.
#include <mutex>

#include "kernels.h"
#include "status.h"

namespace hy {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;

}  // namespace

hy_status tma_map_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle,
                     const char *who) {
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!g_encode) {
            void *fn = nullptr;
            cudaDriverEntryPointQueryResult q;
            const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
            if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
                return set_error(HY_ERR_CUDA, "%s: cuTensorMapEncodeTiled is not available", who);
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
        }
    }
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = g_encode(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return set_error(HY_ERR_CUDA, "%s: cuTensorMapEncodeTiled failed (%d)", who, (int)r);
    return HY_OK;
}

}  // namespace hy
