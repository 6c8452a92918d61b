// State merge: out = a + b (arXiv 2610.20637, abstract: states are additive
// across chunks).  Elementwise over B*H*stride floats with 128-bit accesses
// and a grid sized to the SM count; bound by HBM (two reads, one write).
#include "common.cuh"
#include "internal.h"

namespace ta {

namespace {

__global__ void __launch_bounds__(256)
merge_kernel(const float4* __restrict__ a, const float4* __restrict__ b, float4* out, int64_t n4) {
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float4 x = a[i], y = b[i];
        out[i] = make_float4(x.x + y.x, x.y + y.y, x.z + y.z, x.w + y.w);
    }
}

}  // namespace

cudaError_t launch_merge(const float* a, const float* b, float* out, int64_t count, int num_sms,
                         cudaStream_t stream) {
    const int64_t n4 = count / 4;  // count is a multiple of 32 (state stride)
    if (n4 == 0) return cudaSuccess;
    int64_t blocks = (n4 + 255) / 256;
    const int64_t cap = (int64_t)num_sms * 8;
    if (blocks > cap) blocks = cap;
    TA_TIMED(stream, "merge_kernel",
             merge_kernel<<<(unsigned)blocks, 256, 0, stream>>>(reinterpret_cast<const float4*>(a),
                                                                reinterpret_cast<const float4*>(b),
                                                                reinterpret_cast<float4*>(out), n4));
    return cudaGetLastError();
}

}  // namespace ta
