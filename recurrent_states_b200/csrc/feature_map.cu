// Step 1 of the path on its own: phi(x) for T vectors (arXiv 2610.20637,
// abstract: each Taylor term factors into a tensor-power inner product).
// Inside the prefill and decode kernels the same descriptors are evaluated
// in place; this kernel exposes them so the packed order and the weights can
// be checked on the device.  One CTA per 32 vectors; each thread owns one
// feature column and unranks it once.
#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"

namespace ta {

namespace {

constexpr int kVec = 32;

__global__ void __launch_bounds__(256)
feature_map_kernel(const float* __restrict__ x, float* __restrict__ phi, int64_t T, int d, int n,
                   float tau, int query_side, int64_t F) {
    __shared__ float xs[kVec][kMaxDk];
    __shared__ float qc[kMaxN];
    if (threadIdx.x < n) qc[threadIdx.x] = query_coeff(threadIdx.x, tau);
    const PackedFeat* tab = feat_table(d, n);
    const int64_t t0 = (int64_t)blockIdx.x * kVec;
    const int nv = (int)min64(kVec, T - t0);
    for (int i = threadIdx.x; i < nv * d; i += blockDim.x) xs[i / d][i % d] = x[t0 * d + i];
    __syncthreads();
    for (int64_t f = threadIdx.x + (int64_t)blockIdx.y * blockDim.x; f < F;
         f += (int64_t)gridDim.y * blockDim.x) {
        const FeatDesc fd = get_desc(tab, d, n, f, tau, qc, query_side != 0);
        for (int i = 0; i < nv; ++i) phi[(t0 + i) * F + f] = eval_desc(fd, xs[i]);
    }
}

}  // namespace

cudaError_t launch_feature_map(const float* x, float* phi, int64_t T, int d, int n, float tau,
                               int query_side, int64_t F, cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    const int64_t gx = (T + kVec - 1) / kVec;
    int64_t gy = (F + 255) / 256;
    if (gy > 64) gy = 64;
    if (gx > 0x7fffffff) return cudaErrorInvalidValue;
    TA_TIMED(stream, "feature_map_kernel",
             feature_map_kernel<<<dim3((unsigned)gx, (unsigned)gy), 256, 0, stream>>>(x, phi, T, d, n,
                                                                                     tau, query_side, F));
    return cudaGetLastError();
}

}  // namespace ta
