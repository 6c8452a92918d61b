// Host-side TMA tensor maps (cuTensorMapEncodeTiled, reached through the
// runtime's driver entry point so that the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ta {

// A bf16 tensor [d2][d1][d0] (d0 innermost, contiguous) with boxes of
// box0 x box1 x 1 elements and zero fill outside the tensor.  swizzle_bytes
// 0 (none), 32, 64 or 128: the box's rows (box0 * 2 bytes, at most that many)
// are written with their 16-byte chunks permuted by address bits 7...
// Returns cudaErrorInvalidValue when the driver rejects the description.
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                              uint32_t box0, uint32_t box1, uint32_t swizzle_bytes);

// An fp32 tensor [d2][d1][d0] (d0 innermost, contiguous) with row strides
// stride1 and stride2 bytes (multiples of 16), boxes of box0 x box1 x 1
// elements, and the swizzle as above (box0 * 4 bytes at most that many).
cudaError_t make_tmap_f32_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                             uint64_t stride1, uint64_t stride2, uint32_t box0, uint32_t box1,
                             uint32_t swizzle_bytes);

}  // namespace ta
