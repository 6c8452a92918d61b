// Host-side TMA tensor maps; see tmap.h.
#include "tmap.h"

#include <cudaTypedefs.h>

#include <mutex>

namespace ta {

namespace {
std::once_flag g_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t make_tmap_3d(CUtensorMap* map, CUtensorMapDataType type, const void* base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1,
                         uint32_t swizzle_bytes) {
    std::call_once(g_once, []() {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return cudaErrorNotSupported;
    CUtensorMapSwizzle sw;
    switch (swizzle_bytes) {
        case 0: sw = CU_TENSOR_MAP_SWIZZLE_NONE; break;
        case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
        case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
        case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
        default: return cudaErrorInvalidValue;
    }
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {stride1, stride2};  // bytes, dims 1 and 2
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = g_encode(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}
}  // namespace

cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t box0, uint32_t box1, uint32_t swizzle_bytes) {
    return make_tmap_3d(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, d0, d1, d2, d0 * 2, d0 * d1 * 2, box0, box1,
                        swizzle_bytes);
}

cudaError_t make_tmap_f32_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                             uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1,
                             uint32_t swizzle_bytes) {
    return make_tmap_3d(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, d0, d1, d2, stride1, stride2, box0, box1,
                        swizzle_bytes);
}

}  // namespace ta
