// Decode step of causal attention with the mean-centred Taylor expansion of
// softmax (first or second order), carried in the n = 3 Taylor-kernel state.
//
// Source: Su Jianlin, "Taylor expansions of logsumexp and softmax" (kexue.fm,
// English translation 11814), section "Calculating the Gradient": about the
// mean score, softmax(x) = (1/n)(1 + y + (y^2 - mean(y^2))/2 + ...) with
// y = x - mean(x); section "Linear Attention": on scores x_j = q.k_j the
// truncation is linear attention again, the square being a Frobenius product
// of q q^T with the centred outer product of the keys.
//
// The prefix sums that form needs (n, sum k, sum v, sum k v^T, sum k k^T and
// sum (k k^T) v^T) are the degree-0, 1 and 2 blocks of the n = 3 state
// S = sum phi(k)[v | 1]^T, read through phi_m(q) because
// phi_2(q).phi_2(k) = (q.k)^2.  So the step updates S exactly as the Taylor
// decode does, takes the three per-degree read-outs R_m = phi_m(q)^T S_m
// (multinomial weights only, no tau), and combines them per output column:
//   n = R_0[z], V = R_0[v], qkbar = R_1[z] / n,
//   sum a v   = tau (R_1[v] - qkbar V),
//   sum a^2 v = tau^2 (R_2[v] - 2 qkbar R_1[v] + qkbar^2 V),
//   sum a^2   = tau^2 (R_2[z] - n qkbar^2),
//   o = V/n + (sum a v)/n  [+ (sum a^2 v - (sum a^2) V/n) / (2n) at order 2].
//
// One CTA per head, 256 threads: the token and both feature vectors go to
// shared memory, then each thread streams its rows of S through registers
// with 128-bit loads and stores (one 16-byte column group per row), keeping
// one accumulator per degree; the z column and the column partials are
// reduced in shared memory.
#include "common.cuh"
#include "internal.h"

namespace ta {

namespace {

constexpr int kThreadsC = 256;

template <typename Tin>
__global__ void __launch_bounds__(kThreadsC)
centred_decode_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                      float* __restrict__ state, float* __restrict__ out, int d, int dv, int F, int64_t stride,
                      int order, float tau) {
    extern __shared__ float smc[];
    __shared__ float xq[kMaxDk], xk[kMaxDk], xv[kMaxDv];
    __shared__ float zred[kThreadsC / 32][3];
    const int dv4 = dv >> 2, nrs = kThreadsC / dv4;
    float* pk = smc;           // phi(k)[F]
    float* pq = pk + F;        // phi(q)[F], no tau
    float* red = pq + F;       // [3][nrs][dv] column partials per degree
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t h = blockIdx.x;
    float* S = state + h * stride;
    // the head's state starts towards L2 while the token and the features
    // are prepared (16-byte aligned: the stride is a multiple of 32 floats)
    if (tid == 0) {
        const uint32_t bytes = (uint32_t)(((int64_t)F * (dv + 1) * 4 + 15) / 16 * 16);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(S), "r"(bytes) : "memory");
    }

    for (int i = tid; i < d; i += kThreadsC) {
        xq[i] = to_float(q[h * d + i]);
        xk[i] = to_float(k[h * d + i]);
    }
    for (int i = tid; i < dv; i += kThreadsC) xv[i] = to_float(v[h * dv + i]);
    __syncthreads();
    for (int f = tid; f < F; f += kThreadsC) {
        int m, i, j;
        float w;
        feature_deg2(d, f, m, i, j, w);
        pk[f] = w * (m >= 1 ? xk[i] : 1.0f) * (m >= 2 ? xk[j] : 1.0f);
        pq[f] = w * (m >= 1 ? xq[i] : 1.0f) * (m >= 2 ? xq[j] : 1.0f);
    }
    __syncthreads();

    const int cg = tid % dv4, rs = tid / dv4;
    if (rs < nrs) {
        const float4 v4 = make_float4(xv[4 * cg], xv[4 * cg + 1], xv[4 * cg + 2], xv[4 * cg + 3]);
        float4* S4 = reinterpret_cast<float4*>(S);
        // rows [lo, hi) of one degree whose index is rs modulo nrs
        auto walk = [&](int lo, int hi) -> float4 {
            float4 A = make_float4(0.f, 0.f, 0.f, 0.f);
            const int r0 = lo + ((rs - lo) % nrs + nrs) % nrs;
#pragma unroll 4
            for (int r = r0; r < hi; r += nrs) {
                const float a = pk[r], c = pq[r];
                float4 s = S4[(int64_t)r * dv4 + cg];
                s.x = fmaf(a, v4.x, s.x);
                s.y = fmaf(a, v4.y, s.y);
                s.z = fmaf(a, v4.z, s.z);
                s.w = fmaf(a, v4.w, s.w);
                S4[(int64_t)r * dv4 + cg] = s;
                A.x = fmaf(c, s.x, A.x);
                A.y = fmaf(c, s.y, A.y);
                A.z = fmaf(c, s.z, A.z);
                A.w = fmaf(c, s.w, A.w);
            }
            return A;
        };
        const float4 a0 = walk(0, 1), a1 = walk(1, d + 1), a2 = walk(d + 1, F);
        const float4 acc[3] = {a0, a1, a2};
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            float* dst = red + ((int64_t)m * nrs + rs) * dv + 4 * cg;
            dst[0] = acc[m].x;
            dst[1] = acc[m].y;
            dst[2] = acc[m].z;
            dst[3] = acc[m].w;
        }
    }
    // the normaliser column z, after the rows S_v
    float zr[3] = {0.f, 0.f, 0.f};
    float* Z = S + (int64_t)F * dv;
    for (int r = tid; r < F; r += kThreadsC) {
        const float z = Z[r] + pk[r];
        Z[r] = z;
        const float p = pq[r] * z;
        if (r == 0) zr[0] += p;
        else if (r <= d) zr[1] += p;
        else zr[2] += p;
    }
#pragma unroll
    for (int m = 0; m < 3; ++m)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) zr[m] += __shfl_xor_sync(0xffffffffu, zr[m], o);
    if (lane == 0)
        for (int m = 0; m < 3; ++m) zred[warp][m] = zr[m];
    __syncthreads();

    if (tid < dv) {
        float R[3] = {0.f, 0.f, 0.f}, Rz[3] = {0.f, 0.f, 0.f};
#pragma unroll
        for (int m = 0; m < 3; ++m) {
            for (int s = 0; s < nrs; ++s) R[m] += red[((int64_t)m * nrs + s) * dv + tid];
            for (int w = 0; w < kThreadsC / 32; ++w) Rz[m] += zred[w][m];
        }
        const float n = Rz[0], V = R[0], qkbar = Rz[1] / n;
        float o = V / n + tau * (R[1] - qkbar * V) / n;
        if (order >= 2) {
            const float t2 = tau * tau;
            const float sum_a2v = t2 * (R[2] - 2.0f * qkbar * R[1] + qkbar * qkbar * V);
            const float sum_a2 = t2 * (Rz[2] - n * qkbar * qkbar);
            o += (sum_a2v - sum_a2 * V / n) / (2.0f * n);
        }
        out[h * dv + tid] = o;
    }
}

}  // namespace

template <typename Tin>
cudaError_t launch_centred_decode(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH,
                                  int d, int dv, int order, float tau, int64_t F, int64_t stride,
                                  cudaStream_t stream) {
    if (d < 1 || d > kMaxDk || dv < 4 || dv > kMaxDv || dv % 4 != 0) return cudaErrorNotSupported;
    {  // many heads of a small state: the persistent warp-specialised kernel
        const cudaError_t e = launch_centred_decode_ws(q, k, v, state, out, BH, d, dv, order, tau, F, stride, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    const int nrs = kThreadsC / (dv / 4);
    const size_t smem = (size_t)(2 * F + 3 * (int64_t)nrs * dv) * sizeof(float);
    if (smem > 48 * 1024) return cudaErrorNotSupported;  // F <= 2145 (d_k 64) needs 29.4 KB
    TA_TIMED(stream, "centred_decode_kernel",
             centred_decode_kernel<Tin><<<BH, kThreadsC, smem, stream>>>(q, k, v, state, out, d, dv, (int)F,
                                                                         stride, order, tau));
    return cudaGetLastError();
}

template cudaError_t launch_centred_decode<float>(const float*, const float*, const float*, float*, float*, int,
                                                  int, int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_centred_decode<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                          const __nv_bfloat16*, float*, float*, int, int, int,
                                                          int, float, int64_t, int64_t, cudaStream_t);

}  // namespace ta
