// Device-side error word.  Kernels that wait on an mbarrier (or any other
// asynchronous event) bound the wait; when the bound runs out they OR a bit
// into this word and return without touching their outputs further.  The
// host reads and clears it through taylor_attn_device_errors().
#include <mutex>

#include "../../include/taylor_attn.h"
#include "internal.h"

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
