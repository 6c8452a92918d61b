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

// The whole prefill in one cooperative launch (prefill_fused.cu): d_k 16,
// n <= 3, d_v 64, at most 36 chunks of 128 tokens per head, when every CTA of
// the call (one or two chunks each) can be resident at once; else
// kNotApplicable.
int try_prefill_fused(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream);

// Feature-tiled variant for d_k in {16, 32, 64}, d_v = 64 and any number of
// features (tiles of 128 features; prefill_tcf.cu).
int try_prefill_tiled(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream);

// The mean-centred softmax expansion's prefill (orders 1 and 2) on the tensor
// cores: d_k 16, d_v 64 (the n = 3 state, F = 153); else kNotApplicable.
int try_centred_prefill(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                        float* state_out, int BH, int N, int d, int dv, int order, float tau, int64_t F,
                        int64_t stride, cudaStream_t stream);

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
inline int try_centred_prefill(const float*, const float*, const float*, float*, float*, int, int, int, int, int,
                               float, int64_t, int64_t, cudaStream_t) {
    return kNotApplicable;
}

}  // namespace tc
}  // namespace ta
