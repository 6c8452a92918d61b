// Explicit instantiations of the feature-tiled prefill: (d_k 32, n 1), (d_k 32, n 2), (d_k 32, n 3), (d_k 32, n run-time).
#include "prefill_tcf.cuh"

namespace ta {
namespace tc {
namespace tcf {
template int run<32, 1>(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, const float*, float*, int,
                           int, int, float, int64_t, int64_t, unsigned int*, cudaStream_t);
template int run<32, 2>(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, const float*, float*, int,
                           int, int, float, int64_t, int64_t, unsigned int*, cudaStream_t);
template int run<32, 3>(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, const float*, float*, int,
                           int, int, float, int64_t, int64_t, unsigned int*, cudaStream_t);
template int run<32, 0>(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, const float*, float*, int,
                           int, int, float, int64_t, int64_t, unsigned int*, cudaStream_t);
}  // namespace tcf
}  // namespace tc
}  // namespace ta
