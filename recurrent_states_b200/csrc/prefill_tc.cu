// Tensor-core prefill specialisations (tcgen05, sm_100a).
#include "prefill_tc.h"

namespace ta {
namespace tc {

int try_prefill(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, float*, float*, int,
                int, int, int, int, float, int64_t, int64_t, cudaStream_t) {
    return kNotApplicable;
}

}  // namespace tc
}  // namespace ta
