// Dispatch of the feature-tiled tensor-core prefill (kernels in
// prefill_tcf.cuh; each (d_k, n) specialisation is compiled in its own
// translation unit, tcf_inst_*.cu, so that the build runs them in parallel).
#include "../../include/taylor_attn.h"
#include "internal.h"
#include "prefill_tc.h"

namespace ta {
namespace tc {
namespace tcf {
template <int D, int N>
int run(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out, const float* state_in,
        float* state_out, int BH, int Ntok, int n, float tau, int64_t F, int64_t stride, unsigned int* err,
        cudaStream_t stream);
}  // namespace tcf

int try_prefill_tiled(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream) {
    if (dv != 64 || N <= 0 || BH <= 0) return kNotApplicable;
    unsigned int* err = device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;
#define TA_TCF(DD, NN) return tcf::run<DD, NN>(q, k, v, out, state_in, state_out, BH, N, n, tau, F, stride, err, stream)
    switch (d) {
        case 16:
            if (n == 4) TA_TCF(16, 4);
            if (n == 5) TA_TCF(16, 5);
            TA_TCF(16, 0);
        case 32:
            if (n == 1) TA_TCF(32, 1);
            if (n == 2) TA_TCF(32, 2);
            if (n == 3) TA_TCF(32, 3);
            TA_TCF(32, 0);
        case 64:
            if (n == 1) TA_TCF(64, 1);
            if (n == 2) TA_TCF(64, 2);
            if (n == 3) TA_TCF(64, 3);
            TA_TCF(64, 0);
        default:
            return kNotApplicable;
    }
#undef TA_TCF
}

}  // namespace tc
}  // namespace ta
