// Constant-cost decode step (arXiv 2610.20637, abstract: per-token decoding
// latency is constant in N).  Per (b, h): S += phi(k) [v | 1]^T, then
// y = (c (.) phi(q))^T S and o = y[0:d_v] / y[d_v].
//
// The step is bound by HBM: each head's fp32 state (F*(d_v+1) floats) is read
// once and written once.  One CTA per head; each thread owns one 16-byte
// column group of the S_v rows it visits, so a warp moves whole 128-byte
// lines with 128-bit loads and stores.  The state rows of a thread are loaded
// into registers before the feature map is evaluated, so the loads are in
// flight while phi(q), phi(k) are computed.  The read-out sum over rows is a
// shared-memory reduction across row sets; the normaliser's sum over z is a
// warp-shuffle reduction.
#include "common.cuh"
#include "internal.h"

namespace ta {

namespace {

constexpr int kThreads = 256;
constexpr int kFeatTile = 1024;  // features whose phi(q), phi(k) sit in smem at once
constexpr int kRows = 10;        // S_v rows per thread held in registers per batch

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
              float* __restrict__ state, float* __restrict__ out, int d, int dv, int n,
              float tau, int F, int64_t stride) {
    __shared__ float xs_q[kMaxDk], xs_k[kMaxDk], vs[kMaxDv];
    __shared__ float pk[kFeatTile], pq[kFeatTile];
    __shared__ float4 red[kThreads];
    __shared__ float zred[kThreads / 32];

    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int dv4 = dv >> 2;
    const int rsets = kThreads / dv4;      // row sets (threads sharing a column group)
    const int cg = tid % dv4;
    const int rs = tid / dv4;
    const bool active = rs < rsets;

    float* Sv = state + (int64_t)bh * stride;
    float* Z = Sv + (int64_t)F * dv;

    for (int i = tid; i < d; i += kThreads) {
        xs_q[i] = ldf(q + (int64_t)bh * d + i);
        xs_k[i] = ldf(k + (int64_t)bh * d + i);
    }
    for (int i = tid; i < dv; i += kThreads) vs[i] = ldf(v + (int64_t)bh * dv + i);

    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    float yz = 0.f;

    for (int fb = 0; fb < F; fb += kFeatTile) {
        const int fe = min(F, fb + kFeatTile);
        // first batch of rows: issue the loads before the feature map
        float4 s[kRows];
        float zz[kFeatTile / kThreads];
        int r0 = fb + rs;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            const int r = r0 + i * rsets;
            if (active && r < fe) s[i] = *reinterpret_cast<const float4*>(Sv + (int64_t)r * dv + cg * 4);
        }
#pragma unroll
        for (int i = 0; i < kFeatTile / kThreads; ++i) {
            const int f = fb + tid + i * kThreads;
            if (f < fe) zz[i] = Z[f];
        }
        __syncthreads();  // xs_q, xs_k, vs ready; previous tile's pk/pq consumed
        for (int f = fb + tid; f < fe; f += kThreads) {
            const FeatDesc dk = make_desc(d, n, f, tau, false);
            const FeatDesc dq = make_desc(d, n, f, tau, true);
            pk[f - fb] = eval_desc(dk, xs_k);
            pq[f - fb] = eval_desc(dq, xs_q);
        }
        __syncthreads();
        const float4 v4 = active ? *reinterpret_cast<const float4*>(vs + cg * 4) : make_float4(0, 0, 0, 0);
        for (;;) {
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                const int r = r0 + i * rsets;
                if (active && r < fe) {
                    const float a = pk[r - fb], b = pq[r - fb];
                    float4 t = s[i];
                    t.x = fmaf(a, v4.x, t.x);
                    t.y = fmaf(a, v4.y, t.y);
                    t.z = fmaf(a, v4.z, t.z);
                    t.w = fmaf(a, v4.w, t.w);
                    *reinterpret_cast<float4*>(Sv + (int64_t)r * dv + cg * 4) = t;
                    y.x = fmaf(b, t.x, y.x);
                    y.y = fmaf(b, t.y, y.y);
                    y.z = fmaf(b, t.z, y.z);
                    y.w = fmaf(b, t.w, y.w);
                }
            }
            r0 += kRows * rsets;
            if (r0 >= fe) break;
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                const int r = r0 + i * rsets;
                if (active && r < fe) s[i] = *reinterpret_cast<const float4*>(Sv + (int64_t)r * dv + cg * 4);
            }
        }
#pragma unroll
        for (int i = 0; i < kFeatTile / kThreads; ++i) {
            const int f = fb + tid + i * kThreads;
            if (f < fe) {
                const float z = zz[i] + pk[f - fb];
                Z[f] = z;
                yz = fmaf(pq[f - fb], z, yz);
            }
        }
    }

    // reduce y over row sets, yz over the block
    red[tid] = y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) yz += __shfl_xor_sync(0xffffffffu, yz, o);
    if ((tid & 31) == 0) zred[tid >> 5] = yz;
    __syncthreads();
    if (tid < dv) {
        const int g = tid >> 2, c = tid & 3;
        float acc = 0.f;
        for (int r = 0; r < rsets; ++r) {
            const float4 t = red[r * dv4 + g];
            acc += c == 0 ? t.x : c == 1 ? t.y : c == 2 ? t.z : t.w;
        }
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) den += zred[w];
        out[(int64_t)bh * dv + tid] = acc / den;
    }
}

}  // namespace

template <typename Tin>
cudaError_t launch_decode(const Tin* q, const Tin* k, const Tin* v, float* state, float* out,
                          int BH, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                          cudaStream_t stream) {
    if (BH == 0) return cudaSuccess;
    TA_TIMED(stream, "decode_kernel",
             decode_kernel<Tin><<<BH, kThreads, 0, stream>>>(q, k, v, state, out, d, dv, n, tau, (int)F,
                                                             stride));
    return cudaGetLastError();
}

template cudaError_t launch_decode<float>(const float*, const float*, const float*, float*, float*,
                                          int, int, int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_decode<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                  const __nv_bfloat16*, float*, float*, int, int, int,
                                                  int, float, int64_t, int64_t, cudaStream_t);

}  // namespace ta
