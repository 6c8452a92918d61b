// Prefill for callers that cannot allocate device memory.
//
// taylor_attn_prefill_f32 takes its scratch (one fp32 state per group of
// tokens, for the scan across groups) from cudaMallocAsync.  Some callers
// cannot let a library allocate: a plugin inside a host framework that owns
// all device memory through its own allocator, a serving loop that reserves
// every byte up front and treats any allocation as a failure, or code that
// must never return an out-of-memory status half way through a step.  For
// them this file keeps the scratch in one file-scope __device__ array of a
// fixed size, so the call allocates nothing.
//
// The array exists once per GPU that loads this library and stays there until
// the process exits.  Host code cannot use the array's name as a device
// address (it names a host-side stand-in), so the device address is looked up
// with cudaGetSymbolAddress on the first call made while a device is current.
// CUDA loads a library's device code lazily, so that first lookup is also what
// loads the code holding the array and reserves its 16 MiB on the device: make
// the first call during set-up, before the caller reserves the rest of the
// device's memory and before any stream capture.  A lookup that fails (for
// example for want of those 16 MiB) is not remembered; the next call tries
// again.  Every call on a device shares the one array and leaves its contents
// behind; nothing in it has to start at zero, because every element the
// kernels read is written earlier in the same call.  Calls whose work overlaps
// on the GPU (two streams, or two host threads, on one device) race on the
// array and must be serialised by the caller.
#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "internal.h"

namespace {

// 4 Mi floats = 16 MiB of scratch per device.
constexpr int64_t kScratchFloats = int64_t(4) << 20;
static __device__ __align__(256) float g_prefill_scratch[kScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_lookup_mutex;
std::atomic<float*> g_scratch_ptr[kMaxDevices];

// Device address of the array on the current device.  Only a successful
// lookup is kept; after a failure the next call looks it up again.
cudaError_t scratch_on_current_device(float** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    float* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
    if (p == nullptr) {
        std::lock_guard<std::mutex> lock(g_lookup_mutex);
        p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
        if (p == nullptr) {
            void* addr = nullptr;
            e = cudaGetSymbolAddress(&addr, g_prefill_scratch);
            if (e != cudaSuccess) return e;
            p = static_cast<float*>(addr);
            g_scratch_ptr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return cudaSuccess;
}

bool is_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int64_t taylor_attn_prefill_noalloc_scratch_floats(void) { return kScratchFloats; }

extern "C" int taylor_attn_prefill_f32_noalloc(const float* q, const float* k, const float* v,
                                               float* out, float* state_out, int B, int H, int N,
                                               int d_k, int d_v, int n, float tau,
                                               cudaStream_t stream) {
    if (B < 0 || H < 0 || N < 0 || d_k < 0 || d_v < 0 || n < 0) return TAYLOR_ERR_INVALID_ARG;
    if (n < 1 || n > ta::kMaxN || d_k < 1 || d_k > ta::kMaxDk) return TAYLOR_ERR_UNSUPPORTED;
    if (d_v < 4 || d_v > ta::kMaxDv || (d_v % 4) != 0) return TAYLOR_ERR_UNSUPPORTED;
    if (!isfinite(tau)) return TAYLOR_ERR_INVALID_ARG;
    const int64_t BH = (int64_t)B * H;
    if (BH > 65535 || BH * (int64_t)N >= ((int64_t)1 << 31)) return TAYLOR_ERR_UNSUPPORTED;
    if (BH == 0) return TAYLOR_OK;
    const int64_t F = ta::num_features(d_k, n);
    const int64_t stride = (F * (d_v + 1) + 31) / 32 * 32;
    if (state_out && !is_aligned16(state_out)) return TAYLOR_ERR_MISALIGNED;
    if (N == 0) {
        if (!state_out) return TAYLOR_OK;
        return cudaMemsetAsync(state_out, 0, (size_t)BH * stride * sizeof(float), stream) == cudaSuccess
                   ? TAYLOR_OK
                   : TAYLOR_ERR_CUDA;
    }
    if (!q || !k || !v || !out) return TAYLOR_ERR_INVALID_ARG;
    if (!is_aligned16(q) || !is_aligned16(k) || !is_aligned16(v) || !is_aligned16(out))
        return TAYLOR_ERR_MISALIGNED;

    const ta::CcPlan plan = ta::plan_prefill_cc((int)BH, N, d_k, d_v, n, F, stride);
    const bool need_states = plan.NG > 1 || state_out != nullptr;
    if (need_states && BH * plan.NG * stride > kScratchFloats) return TAYLOR_ERR_SCRATCH_LIMIT;
    float* scratch = nullptr;
    const cudaError_t le = scratch_on_current_device(&scratch);
    if (le != cudaSuccess || scratch == nullptr) {
        cudaGetLastError();
        return le == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
    }
    const cudaError_t e = ta::launch_prefill_cc(q, k, v, out, nullptr, state_out, scratch, plan, (int)BH, N,
                                                d_k, d_v, n, tau, F, stride, stream);
    return e == cudaSuccess ? TAYLOR_OK : TAYLOR_ERR_CUDA;
}
