// Device-side error word.  Kernels that wait on an mbarrier (or any other
// asynchronous event) bound the wait; when the bound runs out they OR a bit
// into this word and return without touching their outputs further.  The
// host reads and clears it through taylor_attn_device_errors().
#include <mutex>

#include "../../include/taylor_attn.h"
#include "internal.h"
#include "ptx.cuh"

namespace {

static __device__ unsigned int g_error_word;

constexpr int kMaxDevices = 64;
std::once_flag g_once[kMaxDevices];
unsigned int* g_ptr[kMaxDevices];

}  // namespace

namespace ta {

unsigned int* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return nullptr;
    }
    std::call_once(g_once[dev], [dev]() {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) {
            cudaGetLastError();
            p = nullptr;
        }
        g_ptr[dev] = static_cast<unsigned int*>(p);
    });
    return g_ptr[dev];
}

}  // namespace ta

namespace {

// Waits on an mbarrier that nothing ever arrives on: the bounded wait must run
// out, set its bit and return.
__global__ void selftest_wait_kernel(unsigned int polls, unsigned int* err) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        ta::ptx::mbar_init(&bar, 1);
        ta::ptx::fence_mbar_init();
    }
    __syncthreads();
    const bool done = ta::ptx::mbar_wait(&bar, 0, polls);
    if (!done && threadIdx.x == 0) atomicOr(err, ta::kErrSelfTest);
}

}  // namespace

extern "C" int taylor_attn_selftest_bounded_wait(unsigned int polls, cudaStream_t stream) {
    if (polls == 0 || polls > (1u << 20)) return TAYLOR_ERR_INVALID_ARG;
    unsigned int* err = ta::device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;
    selftest_wait_kernel<<<1, 32, 0, stream>>>(polls, err);
    return cudaGetLastError() == cudaSuccess ? TAYLOR_OK : TAYLOR_ERR_CUDA;
}

extern "C" int taylor_attn_device_errors(int clear, unsigned int* flags) {
    if (!flags) return TAYLOR_ERR_INVALID_ARG;
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_CUDA;
    }
    *flags = v;
    if (clear && v) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_CUDA;
        }
    }
    return v ? TAYLOR_ERR_TIMEOUT : TAYLOR_OK;
}
