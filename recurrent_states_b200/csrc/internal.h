// Launchers shared between the translation units of libtaylor_attn (not part
// of the public ABI).  Each returns the CUDA error of its launch(es).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ta {

// Opt-in per-launch event timing (timing.cu).  TA_TIMED brackets one launch.
namespace timing {
bool enabled();
void begin(cudaStream_t s, const char* name);
void end(cudaStream_t s);
}  // namespace timing

#define TA_TIMED(stream, name, ...)              \
    do {                                         \
        ::ta::timing::begin((stream), (name));   \
        __VA_ARGS__;                             \
        ::ta::timing::end((stream));             \
    } while (0)

// Stream-ordered workspace from the library's per-device pool (workspace.cu).
cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream);
cudaError_t workspace_free(void* ptr, cudaStream_t stream);

// Device address of the error word (errors.cu) on the current device.
unsigned int* device_error_word();
constexpr unsigned int kErrDecodeLoad = 1u;
constexpr unsigned int kErrDecodeStore = 2u;
constexpr unsigned int kErrPrefillPipe = 4u;
constexpr unsigned int kErrSelfTest = 8u;

template <typename Tin>
cudaError_t launch_decode(const Tin* q, const Tin* k, const Tin* v, float* state, float* out,
                          int BH, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                          cudaStream_t stream);

// Decode step of the mean-centred softmax expansion (order 1 or 2) over the
// n = 3 Taylor state (centred.cu).
template <typename Tin>
cudaError_t launch_centred_decode(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH,
                                  int d, int dv, int order, float tau, int64_t F, int64_t stride,
                                  cudaStream_t stream);

// The same persistent kernel with the mean-centred expansion's read-out
// (order 1 or 2) over the n = 3 state; cudaErrorNotSupported as above.
template <typename Tin>
cudaError_t launch_centred_decode_ws(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH,
                                     int d, int dv, int order, float tau, int64_t F, int64_t stride,
                                     cudaStream_t stream);

// Persistent warp-specialised decode for d_v 64 and at most 256 features;
// cudaErrorNotSupported when the shape (or a small number of heads) is
// better served by the one-CTA-per-head kernel.
template <typename Tin>
cudaError_t launch_decode_ws(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH, int d,
                             int dv, int n, float tau, int64_t F, int64_t stride, cudaStream_t stream);

// Batched multi-token decode: T (1..16) new tokens per head against
// state_in, outputs for all of them and (if state_out) the updated state;
// cudaErrorNotSupported when the shape is outside the kernel's range.
template <typename Tin>
cudaError_t launch_decode_multi(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* state_out,
                                float* out, int BH, int T, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                                cudaStream_t stream);

// The same on the tensor cores for bf16 inputs, d_v 64, at most 160 features
// of degree <= 2 and many heads; cudaErrorNotSupported outside that range.
cudaError_t launch_decode_multi_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* state_in, float* state_out, float* out, int BH, int T, int d, int dv,
                                   int n, float tau, int64_t F, int64_t stride, cudaStream_t stream);

cudaError_t launch_merge(const float* a, const float* b, float* out, int64_t count, int num_sms,
                         cudaStream_t stream);

cudaError_t launch_feature_map(const float* x, float* phi, int64_t T, int d, int n, float tau,
                               int query_side, int64_t F, cudaStream_t stream);

// Chunked prefill on CUDA cores (fp32 arithmetic), in three launches:
// per-group states, an exclusive scan over groups, then per-chunk outputs.
struct CcPlan {
    int G;         // tokens per group (multiple of 64)
    int NG;        // groups per head
    size_t ws_bytes;
};
CcPlan plan_prefill_cc(int BH, int N, int d, int dv, int n, int64_t F, int64_t stride);

// In place: W[bh][g] <- state_in[bh] + sum_{g' < g} W[bh][g'] over the first
// `used` floats of each state (state_in may be NULL: zero); state_out[bh]
// (if not NULL) <- the total, zero padded.
cudaError_t launch_state_scan(float* W, const float* state_in, float* state_out, int BH, int NG, int64_t stride,
                              int64_t used, cudaStream_t stream, bool pdl = false);

// Launches `kernel` with programmatic stream serialisation when pdl is set,
// so that it may start while the previous kernel in the stream finishes.
template <typename... KArgs, typename... Args>
cudaError_t launch_maybe_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                             bool pdl, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Prefill of the mean-centred softmax expansion (order 1 or 2) on CUDA cores,
// over the n = 3 group states of the same plan (plan_prefill_cc with n = 3).
template <typename Tin>
cudaError_t launch_centred_prefill_cc(const Tin* q, const Tin* k, const Tin* v, float* out,
                                      const float* state_in, float* state_out, float* workspace,
                                      const CcPlan& plan, int BH, int N, int d, int dv, int order, float tau,
                                      int64_t F, int64_t stride, cudaStream_t stream);

template <typename Tin>
cudaError_t launch_prefill_cc(const Tin* q, const Tin* k, const Tin* v, float* out,
                              const float* state_in, float* state_out, float* workspace,
                              const CcPlan& plan, int BH, int N, int d, int dv, int n, float tau,
                              int64_t F, int64_t stride, cudaStream_t stream);

}  // namespace ta
