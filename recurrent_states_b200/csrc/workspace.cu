// Stream-ordered workspace for the prefill scan.  Each device gets one
// library-owned memory pool whose release threshold keeps freed workspace
// mapped, so back-to-back calls reuse it instead of unmapping and mapping
// memory on every call (which stalls the stream for hundreds of microseconds,
// and for milliseconds at a gigabyte).  The threshold is the larger of
// kCachedBytes and the largest single workspace requested so far on that
// device, so a call whose workspace alone exceeds kCachedBytes still finds it
// mapped on the next call.  taylor_attn_release_workspace() returns the cached
// memory to the driver.
#include <atomic>
#include <mutex>

#include "../../include/taylor_attn.h"
#include "internal.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kCachedBytes = uint64_t(1) << 30;  // 1 GiB per device

std::once_flag g_once[kMaxDevices];
cudaMemPool_t g_pool[kMaxDevices];
cudaError_t g_err[kMaxDevices];
std::atomic<uint64_t> g_threshold[kMaxDevices];
std::mutex g_threshold_mutex;

cudaError_t pool_for(int dev, cudaMemPool_t* out) {
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(g_once[dev], [dev]() {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p = nullptr;
        g_err[dev] = cudaMemPoolCreate(&p, &props);
        if (g_err[dev] == cudaSuccess) {
            uint64_t thr = kCachedBytes;
            g_err[dev] = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
            g_threshold[dev].store(thr);
        }
        g_pool[dev] = p;
    });
    *out = g_pool[dev];
    return g_err[dev];
}

}  // namespace

namespace ta {

cudaError_t workspace_alloc(void** ptr, size_t bytes, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    cudaMemPool_t pool = nullptr;
    if ((e = pool_for(dev, &pool)) != cudaSuccess) return e;
    if (bytes > g_threshold[dev].load(std::memory_order_relaxed)) {
        std::lock_guard<std::mutex> lock(g_threshold_mutex);
        uint64_t thr = bytes;
        if (thr > g_threshold[dev].load()) {
            if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr)) != cudaSuccess) return e;
            g_threshold[dev].store(thr);
        }
    }
    return cudaMallocFromPoolAsync(ptr, bytes, pool, stream);
}

cudaError_t workspace_free(void* ptr, cudaStream_t stream) { return cudaFreeAsync(ptr, stream); }

}  // namespace ta

extern "C" int taylor_attn_release_workspace(void) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_CUDA;
    }
    cudaMemPool_t pool = nullptr;
    if (pool_for(dev, &pool) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemPoolTrimTo(pool, 0) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_CUDA;
    }
    return TAYLOR_OK;
}
