// Host side of the C ABI declared in include/taylor_attn.h: argument checks,
// shape-dependent dispatch and stream-ordered workspace.  No entry point
// prints, throws, exits or synchronises; each returns a status code.
#include <math.h>
#include <stdint.h>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "internal.h"
#include "prefill_tc.h"

namespace {

constexpr int kVersion = 10000;  // 1.0.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Range checks shared by every call; returns TAYLOR_OK or an error code.
int check_dims(int d_k, int d_v, int n) {
    if (d_k < 0 || d_v < 0 || n < 0) return TAYLOR_ERR_INVALID_ARG;
    if (n < 1 || n > ta::kMaxN) return TAYLOR_ERR_UNSUPPORTED;
    if (d_k < 1 || d_k > ta::kMaxDk) return TAYLOR_ERR_UNSUPPORTED;
    if (d_v < 4 || d_v > ta::kMaxDv || (d_v % 4) != 0) return TAYLOR_ERR_UNSUPPORTED;
    return TAYLOR_OK;
}

int64_t stride_of(int d_k, int d_v, int n) {
    const int64_t used = ta::num_features(d_k, n) * (int64_t)(d_v + 1);
    return (used + 31) / 32 * 32;
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TAYLOR_OK;
    if (e == cudaErrorMemoryAllocation) return TAYLOR_ERR_OUT_OF_MEMORY;
    return TAYLOR_ERR_CUDA;
}

int num_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

template <typename Tin>
int prefill_impl(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* out,
                 float* state_out, int B, int H, int N, int d_k, int d_v, int n, float tau,
                 cudaStream_t stream, bool allow_tc) {
    if (B < 0 || H < 0 || N < 0) return TAYLOR_ERR_INVALID_ARG;
    int rc = check_dims(d_k, d_v, n);
    if (rc != TAYLOR_OK) return rc;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    if (BH > 65535) return TAYLOR_ERR_UNSUPPORTED;
    if (BH * (int64_t)N >= ((int64_t)1 << 31)) return TAYLOR_ERR_UNSUPPORTED;
    if (BH == 0) return TAYLOR_OK;
    const int64_t F = ta::num_features(d_k, n);
    const int64_t stride = stride_of(d_k, d_v, n);
    if (state_out && !aligned16(state_out)) return TAYLOR_ERR_MISALIGNED;
    if (state_in && !aligned16(state_in)) return TAYLOR_ERR_MISALIGNED;
    if (N == 0) {
        if (!state_out) return TAYLOR_OK;
        const size_t bytes = (size_t)BH * stride * sizeof(float);
        if (!state_in) return cuda_status(cudaMemsetAsync(state_out, 0, bytes, stream));
        if (state_in == state_out) return TAYLOR_OK;
        return cuda_status(cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, stream));
    }
    if (!q || !k || !v || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TAYLOR_ERR_MISALIGNED;

    if (state_in != nullptr && N <= 16) {
        // a few new tokens against a carried state: one pass over the state
        const cudaError_t e = ta::launch_decode_multi(q, k, v, state_in, state_out, out, (int)BH, N, d_k, d_v, n,
                                                      tau, F, stride, stream);
        if (e != cudaErrorNotSupported) return cuda_status(e);
    }
    if (allow_tc) {
        const int fused = ta::tc::try_prefill_fused(q, k, v, out, state_in, state_out, (int)BH, N, d_k, d_v, n, tau, F,
                                                    stride, stream);
        if (fused != ta::tc::kNotApplicable) return fused;
        const int tc = ta::tc::try_prefill(q, k, v, out, state_in, state_out, (int)BH, N, d_k, d_v, n, tau, F,
                                           stride, stream);
        if (tc != ta::tc::kNotApplicable) return tc;
        const int tcf = ta::tc::try_prefill_tiled(q, k, v, out, state_in, state_out, (int)BH, N, d_k, d_v, n, tau,
                                                  F, stride, stream);
        if (tcf != ta::tc::kNotApplicable) return tcf;
    }

    const ta::CcPlan plan = ta::plan_prefill_cc((int)BH, N, d_k, d_v, n, F, stride);
    float* ws = nullptr;
    const bool need_ws = plan.NG > 1 || state_out != nullptr || state_in != nullptr;
    if (need_ws) {
        cudaError_t e = ta::workspace_alloc(reinterpret_cast<void**>(&ws), plan.ws_bytes, stream);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_OUT_OF_MEMORY;
        }
    }
    cudaError_t e = ta::launch_prefill_cc(q, k, v, out, state_in, state_out, ws, plan, (int)BH, N, d_k,
                                          d_v, n, tau, F, stride, stream);
    if (ws) {
        cudaError_t e2 = ta::workspace_free(ws, stream);
        if (e == cudaSuccess) e = e2;
    }
    return cuda_status(e);
}

template <typename Tin>
int centred_prefill_impl(const Tin* q, const Tin* k, const Tin* v, float* out, float* state_out, int B, int H,
                         int N, int d_k, int d_v, int order, float tau, cudaStream_t stream) {
    if (B < 0 || H < 0 || N < 0) return TAYLOR_ERR_INVALID_ARG;
    int rc = check_dims(d_k, d_v, 3);
    if (rc != TAYLOR_OK) return rc;
    if (order != 1 && order != 2) return TAYLOR_ERR_UNSUPPORTED;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    if (BH > 65535) return TAYLOR_ERR_UNSUPPORTED;
    if (BH * (int64_t)N >= ((int64_t)1 << 31)) return TAYLOR_ERR_UNSUPPORTED;
    if (BH == 0) return TAYLOR_OK;
    const int64_t F = ta::num_features(d_k, 3);
    const int64_t stride = stride_of(d_k, d_v, 3);
    if (state_out && !aligned16(state_out)) return TAYLOR_ERR_MISALIGNED;
    if (N == 0) {
        if (!state_out) return TAYLOR_OK;
        return cuda_status(cudaMemsetAsync(state_out, 0, (size_t)BH * stride * sizeof(float), stream));
    }
    if (!q || !k || !v || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return TAYLOR_ERR_MISALIGNED;
    const int tc = ta::tc::try_centred_prefill(q, k, v, out, state_out, (int)BH, N, d_k, d_v, order, tau, F, stride,
                                               stream);
    if (tc != ta::tc::kNotApplicable) return tc;
    const ta::CcPlan plan = ta::plan_prefill_cc((int)BH, N, d_k, d_v, 3, F, stride);
    float* ws = nullptr;
    if (plan.NG > 1 || state_out != nullptr) {
        if (ta::workspace_alloc(reinterpret_cast<void**>(&ws), plan.ws_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_OUT_OF_MEMORY;
        }
    }
    cudaError_t e = ta::launch_centred_prefill_cc(q, k, v, out, nullptr, state_out, ws, plan, (int)BH, N, d_k, d_v,
                                                  order, tau, F, stride, stream);
    if (ws) {
        const cudaError_t e2 = ta::workspace_free(ws, stream);
        if (e == cudaSuccess) e = e2;
    }
    return cuda_status(e);
}

template <typename Tin>
int decode_impl(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int B, int H,
                int d_k, int d_v, int n, float tau, cudaStream_t stream) {
    if (B < 0 || H < 0) return TAYLOR_ERR_INVALID_ARG;
    int rc = check_dims(d_k, d_v, n);
    if (rc != TAYLOR_OK) return rc;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    if (BH >= ((int64_t)1 << 31)) return TAYLOR_ERR_UNSUPPORTED;
    if (BH == 0) return TAYLOR_OK;
    if (!q || !k || !v || !state || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
        return TAYLOR_ERR_MISALIGNED;
    const int64_t F = ta::num_features(d_k, n);
    return cuda_status(ta::launch_decode(q, k, v, state, out, (int)BH, d_k, d_v, n, tau, F,
                                         stride_of(d_k, d_v, n), stream));
}

template <typename Tin>
int centred_decode_impl(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int B, int H,
                        int d_k, int d_v, int order, float tau, cudaStream_t stream) {
    if (B < 0 || H < 0) return TAYLOR_ERR_INVALID_ARG;
    int rc = check_dims(d_k, d_v, 3);
    if (rc != TAYLOR_OK) return rc;
    if (order != 1 && order != 2) return TAYLOR_ERR_UNSUPPORTED;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    if (BH >= ((int64_t)1 << 31)) return TAYLOR_ERR_UNSUPPORTED;
    if (BH == 0) return TAYLOR_OK;
    if (!q || !k || !v || !state || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
        return TAYLOR_ERR_MISALIGNED;
    const int64_t F = ta::num_features(d_k, 3);
    const cudaError_t e = ta::launch_centred_decode(q, k, v, state, out, (int)BH, d_k, d_v, order, tau, F,
                                                    stride_of(d_k, d_v, 3), stream);
    if (e == cudaErrorNotSupported) return TAYLOR_ERR_UNSUPPORTED;
    return cuda_status(e);
}

}  // namespace

extern "C" {

const char* taylor_attn_strerror(int status) {
    switch (status) {
        case TAYLOR_OK: return "ok";
        case TAYLOR_ERR_INVALID_ARG: return "invalid argument (NULL pointer, negative size or non-finite tau)";
        case TAYLOR_ERR_UNSUPPORTED: return "unsupported size (n, d_k, d_v or total size out of range)";
        case TAYLOR_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case TAYLOR_ERR_CUDA: return "CUDA runtime call or kernel launch failed";
        case TAYLOR_ERR_OUT_OF_MEMORY: return "stream-ordered workspace allocation failed";
        case TAYLOR_ERR_SCRATCH_LIMIT: return "work needs more than the fixed no-alloc scratch";
        case TAYLOR_ERR_TIMEOUT: return "a bounded device-side wait ran out (see taylor_attn_device_errors)";
        default: return "unknown status";
    }
}

int taylor_attn_version(void) { return kVersion; }

int64_t taylor_attn_num_features(int d_k, int n) {
    if (n < 1 || n > ta::kMaxN || d_k < 1 || d_k > ta::kMaxDk) return -1;
    return ta::num_features(d_k, n);
}

int64_t taylor_attn_state_stride(int d_k, int d_v, int n) {
    if (check_dims(d_k, d_v, n) != TAYLOR_OK) return -1;
    return stride_of(d_k, d_v, n);
}

int taylor_attn_feature_index(int d_k, int n, int32_t* deg, int32_t* idx) {
    if (n < 1 || n > ta::kMaxN || d_k < 1 || d_k > ta::kMaxDk) return TAYLOR_ERR_UNSUPPORTED;
    if (!deg || !idx) return TAYLOR_ERR_INVALID_ARG;
    const int64_t F = ta::num_features(d_k, n);
    const int width = n > 1 ? n - 1 : 1;
    for (int64_t f = 0; f < F; ++f) {
        const ta::Mono mo = ta::unrank(d_k, n, f);
        deg[f] = mo.m;
        for (int p = 0; p < width; ++p) idx[f * width + p] = p < mo.m ? mo.idx[p] : -1;
    }
    return TAYLOR_OK;
}

int taylor_attn_feature_map(const float* x, float* phi, int64_t T, int d_k, int n, float tau,
                            int query_side, cudaStream_t stream) {
    if (T < 0) return TAYLOR_ERR_INVALID_ARG;
    if (n < 1 || n > ta::kMaxN || d_k < 1 || d_k > ta::kMaxDk) return TAYLOR_ERR_UNSUPPORTED;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    if (T == 0) return TAYLOR_OK;
    if (!x || !phi) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(phi)) return TAYLOR_ERR_MISALIGNED;
    const int64_t F = ta::num_features(d_k, n);
    return cuda_status(ta::launch_feature_map(x, phi, T, d_k, n, tau, query_side, F, stream));
}

int taylor_attn_prefill(const void* q, const void* k, const void* v, float* out, float* state_out,
                        int B, int H, int N, int d_k, int d_v, int n, float tau, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return prefill_impl(static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
                        nullptr, out, state_out, B, H, N, d_k, d_v, n, tau, stream, true);
}

int taylor_attn_prefill_from_state(const void* q, const void* k, const void* v, const float* state_in,
                                   float* out, float* state_out, int B, int H, int N, int d_k, int d_v,
                                   int n, float tau, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    if (!state_in && B > 0 && H > 0) return TAYLOR_ERR_INVALID_ARG;
    return prefill_impl(static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
                        state_in, out, state_out, B, H, N, d_k, d_v, n, tau, stream, true);
}

int taylor_attn_prefill_from_state_f32(const float* q, const float* k, const float* v, const float* state_in,
                                       float* out, float* state_out, int B, int H, int N, int d_k, int d_v,
                                       int n, float tau, cudaStream_t stream) {
    if (!state_in && B > 0 && H > 0) return TAYLOR_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, state_in, out, state_out, B, H, N, d_k, d_v, n, tau, stream, false);
}

int taylor_attn_prefill_f32(const float* q, const float* k, const float* v, float* out,
                            float* state_out, int B, int H, int N, int d_k, int d_v, int n, float tau,
                            cudaStream_t stream) {
    return prefill_impl(q, k, v, nullptr, out, state_out, B, H, N, d_k, d_v, n, tau, stream, false);
}

int taylor_attn_decode(const void* q, const void* k, const void* v, float* state_inout, float* out,
                       int B, int H, int d_k, int d_v, int n, float tau, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return decode_impl(static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
                       state_inout, out, B, H, d_k, d_v, n, tau, stream);
}

int taylor_attn_decode_f32(const float* q, const float* k, const float* v, float* state_inout,
                           float* out, int B, int H, int d_k, int d_v, int n, float tau,
                           cudaStream_t stream) {
    return decode_impl(q, k, v, state_inout, out, B, H, d_k, d_v, n, tau, stream);
}

int taylor_attn_centred_decode(const void* q, const void* k, const void* v, float* state_inout, float* out,
                               int B, int H, int d_k, int d_v, int order, float tau, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return centred_decode_impl(static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
                               state_inout, out, B, H, d_k, d_v, order, tau, stream);
}

int taylor_attn_centred_decode_f32(const float* q, const float* k, const float* v, float* state_inout,
                                   float* out, int B, int H, int d_k, int d_v, int order, float tau,
                                   cudaStream_t stream) {
    return centred_decode_impl(q, k, v, state_inout, out, B, H, d_k, d_v, order, tau, stream);
}

int taylor_attn_centred_prefill(const void* q, const void* k, const void* v, float* out, float* state_out, int B,
                                int H, int N, int d_k, int d_v, int order, float tau, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    return centred_prefill_impl(static_cast<const bf*>(q), static_cast<const bf*>(k), static_cast<const bf*>(v),
                                out, state_out, B, H, N, d_k, d_v, order, tau, stream);
}

int taylor_attn_centred_prefill_f32(const float* q, const float* k, const float* v, float* out, float* state_out,
                                    int B, int H, int N, int d_k, int d_v, int order, float tau,
                                    cudaStream_t stream) {
    return centred_prefill_impl(q, k, v, out, state_out, B, H, N, d_k, d_v, order, tau, stream);
}

int taylor_attn_state_merge(const float* a, const float* b, float* out, int B, int H, int d_k,
                            int d_v, int n, cudaStream_t stream) {
    if (B < 0 || H < 0) return TAYLOR_ERR_INVALID_ARG;
    int rc = check_dims(d_k, d_v, n);
    if (rc != TAYLOR_OK) return rc;
    const int64_t BH = (int64_t)B * H;
    if (BH == 0) return TAYLOR_OK;
    if (!a || !b || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!aligned16(a) || !aligned16(b) || !aligned16(out)) return TAYLOR_ERR_MISALIGNED;
    return cuda_status(ta::launch_merge(a, b, out, BH * stride_of(d_k, d_v, n), num_sms(), stream));
}

}  // extern "C"
