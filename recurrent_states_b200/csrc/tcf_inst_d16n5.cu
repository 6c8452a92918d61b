// Explicit instantiations of the feature-tiled prefill: (d_k 16, n 5).
#include "prefill_tcf.cuh"

namespace ta {
namespace tc {
namespace tcf {
template int run<16, 5>(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, const float*, float*, int,
                           int, int, float, int64_t, int64_t, unsigned int*, cudaStream_t);
}  // namespace tcf
}  // namespace tc
}  // namespace ta
