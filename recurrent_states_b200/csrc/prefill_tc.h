// Tensor-core (tcgen05) prefill specialisations.  try_prefill returns
// kNotApplicable when no specialisation covers the shape, else a
// taylor_attn status.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ta {
namespace tc {

constexpr int kNotApplicable = 1;

int try_prefill(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                int64_t F, int64_t stride, cudaStream_t stream);

// Feature-tiled variant for d_k in {16, 32, 64}, d_v = 64 and any number of
// features (tiles of 128 features; prefill_tcf.cu).
// The whole prefill in one cluster launch (prefill_fused.cu): d_k 16, n <= 3,
// d_v 64 and at most 16 x 256 tokens per head, on devices that can host a
// cluster of the needed size; else kNotApplicable.
int try_prefill_fused(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream);

int try_prefill_tiled(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream);

// fp32 inputs never take the tensor-core path.
inline int try_prefill(const float*, const float*, const float*, float*, const float*, float*, int, int, int,
                       int, int, float, int64_t, int64_t, cudaStream_t) {
    return kNotApplicable;
}
inline int try_prefill_tiled(const float*, const float*, const float*, float*, const float*, float*, int, int,
                             int, int, int, float, int64_t, int64_t, cudaStream_t) {
    return kNotApplicable;
}
inline int try_prefill_fused(const float*, const float*, const float*, float*, const float*, float*, int, int,
                             int, int, int, float, int64_t, int64_t, cudaStream_t) {
    return kNotApplicable;
}

}  // namespace tc
}  // namespace ta
