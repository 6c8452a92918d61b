// Several new tokens per head against a carried state in one pass over the
// state (batched multi-token decode): the decode step of the paper (arXiv
// 2610.20637, abstract: constant per-token cost, the history held in the
// additive states) generalised to a block of T <= 16 tokens, with the
// block's own causal part computed pairwise.  For token i of the block,
//   y_i = (c (.) phi(q_i))^T S_prev + sum_{j <= i in the block} K(q_i, k_j) [v_j | 1],
//   o_i = y_i[0:d_v] / y_i[d_v],
// and the state leaves as S_prev + sum_j phi(k_j) [v_j | 1]^T.
//
// state_out may alias state_in (update in place): the whole state is in
// shared memory before the first store.  One CTA per head.  One thread
// brings the head's state into shared memory with a bulk copy while every
// thread loads the block's tokens and evaluates
// phi(k_j), phi(q_i) and the pairwise K(q_i, k_j); then each thread walks its
// state rows once (one 16-byte column group per row), accumulating the
// read-out of all T tokens from the old row, adding the T rank-one updates
// and storing the new row straight to HBM.  HBM traffic is one state read and
// one state write per call, as for a single decode step.
#include <mutex>

#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace ta {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTMax = 16;
constexpr uint32_t kWaitPolls = 1u << 22;
constexpr size_t kMaxDyn = 226 * 1024;  // the 227 KB per-block limit, less static shared memory
constexpr int kMaxDevices = 64;

struct MultiLayout {
    uint32_t s, pk, pq, xq, xk, vv, p, red, zr, bytes;
};

// phi(k_j), phi(q_i) are stored feature-major with the block's tokens
// contiguous ([F][Tp], Tp = T rounded up to 4, zero padded), so that the row
// loop reads the coefficients of four tokens with one 16-byte load.
__host__ __device__ inline MultiLayout multi_layout(int T, int d, int dv, int F, uint32_t state_bytes) {
    auto al = [](uint32_t x) { return (x + 127u) & ~127u; };
    const uint32_t Tp = (uint32_t)((T + 3) & ~3);
    MultiLayout L;
    L.s = 0;
    L.pk = al(state_bytes);
    L.pq = L.pk + al((uint32_t)F * Tp * 4);
    L.xq = L.pq + al((uint32_t)F * Tp * 4);
    L.xk = L.xq + al((uint32_t)(T * d) * 4);
    L.vv = L.xk + al((uint32_t)(T * d) * 4);
    L.p = L.vv + al((uint32_t)(T * dv) * 4);
    L.red = L.p + al((uint32_t)(kTMax * kTMax) * 4);
    L.zr = L.red + al((uint32_t)(kWarps * T * dv) * 4);
    L.bytes = L.zr + al((uint32_t)(kWarps * T) * 4);
    return L;
}

template <typename Tin, int DV4>
__global__ void __launch_bounds__(kThreads)
decode_multi_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                    const float* state_in, float* state_out, float* __restrict__ out, int T,
                    int d, int n, float tau, int F, int64_t stride, uint32_t bytes, unsigned int* __restrict__ err) {
    constexpr int DV = DV4 * 4;
    constexpr int RS = kThreads / DV4;  // row sets
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ float qc[kMaxN];
    const MultiLayout L = multi_layout(T, d, DV, F, bytes);
    const int Tp = (T + 3) & ~3;
    const float* S = reinterpret_cast<const float*>(dsm + L.s);
    float* pk = reinterpret_cast<float*>(dsm + L.pk);
    float* pq = reinterpret_cast<float*>(dsm + L.pq);
    float* xq = reinterpret_cast<float*>(dsm + L.xq);
    float* xk = reinterpret_cast<float*>(dsm + L.xk);
    float* vv = reinterpret_cast<float*>(dsm + L.vv);
    float* P = reinterpret_cast<float*>(dsm + L.p);
    float4* red = reinterpret_cast<float4*>(dsm + L.red);
    float* zr = reinterpret_cast<float*>(dsm + L.zr);

    const int bh = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_arrive_expect_tx(&bar, bytes);
        ptx::bulk_g2s(dsm + L.s, state_in + (int64_t)bh * stride, bytes, &bar);
    }
    const int64_t tok0 = (int64_t)bh * T;
    for (int e = tid; e < T * d; e += kThreads) {
        xq[e] = ldf(q + tok0 * d + e);
        xk[e] = ldf(k + tok0 * d + e);
    }
    for (int e = tid; e < T * DV; e += kThreads) vv[e] = ldf(v + tok0 * DV + e);
    if (tid < n) qc[tid] = query_coeff(tid, tau);
    __syncthreads();
    const PackedFeat* tab = feat_table(d, n);
    for (int f = tid; f < F; f += kThreads) {  // one descriptor load per feature, all tokens
        const FeatDesc dk = tab ? desc_from_packed(tab[f], qc, false) : make_desc(d, n, f, tau, false);
        const FeatDesc dq = tab ? desc_from_packed(tab[f], qc, true) : make_desc(d, n, f, tau, true);
        for (int j = 0; j < Tp; ++j) {
            pk[f * Tp + j] = j < T ? eval_desc(dk, xk + j * d) : 0.f;
            pq[f * Tp + j] = j < T ? eval_desc(dq, xq + j * d) : 0.f;
        }
    }
    for (int e = tid; e < T * T; e += kThreads) {
        const int i = e / T, j = e % T;
        float w = 0.f;
        if (j <= i) {
            float dot = 0.f;
            for (int c = 0; c < d; ++c) dot = fmaf(xq[i * d + c], xk[j * d + c], dot);
            w = taylor_kernel(tau * dot, n);
        }
        P[i * kTMax + j] = w;
    }
    const bool landed = ptx::mbar_wait(&bar, 0, kWaitPolls);
    if (!__syncthreads_and(landed)) {
        if (tid == 0) atomicOr(err, kErrDecodeLoad);
        if (!landed) ptx::mbar_wait(&bar, 0, kWaitPolls);  // one more bound for the copy in flight
        return;
    }

    // rows: read-out of every token from the old row, then the T updates
    const int cg = tid % DV4, rs = tid / DV4;
    const float4* S4 = reinterpret_cast<const float4*>(S);
    const float4* V4 = reinterpret_cast<const float4*>(vv);
    float4* G4 = state_out ? reinterpret_cast<float4*>(state_out + (int64_t)bh * stride) : nullptr;
    float4 y[kTMax];
#pragma unroll
    for (int i = 0; i < kTMax; ++i) y[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fma4 = [](float c, const float4& a, float4& acc) {
        acc.x = fmaf(c, a.x, acc.x);
        acc.y = fmaf(c, a.y, acc.y);
        acc.z = fmaf(c, a.z, acc.z);
        acc.w = fmaf(c, a.w, acc.w);
    };
    for (int r = rs; r < F; r += RS) {
        float4 s = S4[r * DV4 + cg];
        const float4* cq = reinterpret_cast<const float4*>(pq + r * Tp);
#pragma unroll
        for (int i4 = 0; i4 < kTMax / 4; ++i4) {
            if (4 * i4 < T) {
                const float4 c = cq[i4];
                fma4(c.x, s, y[4 * i4]);
                fma4(c.y, s, y[4 * i4 + 1]);
                fma4(c.z, s, y[4 * i4 + 2]);
                fma4(c.w, s, y[4 * i4 + 3]);
            }
        }
        if (G4) {
            const float4* ck = reinterpret_cast<const float4*>(pk + r * Tp);
#pragma unroll
            for (int j4 = 0; j4 < kTMax / 4; ++j4) {
                if (4 * j4 < T) {  // padded tokens have coefficient 0 (and finite v rows)
                    const float4 a = ck[j4];
                    fma4(a.x, V4[(4 * j4) * DV4 + cg], s);
                    if (4 * j4 + 1 < T) fma4(a.y, V4[(4 * j4 + 1) * DV4 + cg], s);
                    if (4 * j4 + 2 < T) fma4(a.z, V4[(4 * j4 + 2) * DV4 + cg], s);
                    if (4 * j4 + 3 < T) fma4(a.w, V4[(4 * j4 + 3) * DV4 + cg], s);
                }
            }
            G4[r * DV4 + cg] = s;
        }
    }
    float yz[kTMax];
#pragma unroll
    for (int i = 0; i < kTMax; ++i) yz[i] = 0.f;
    const float* Z = S + (int64_t)F * DV;
    float* GZ = state_out ? state_out + (int64_t)bh * stride + (int64_t)F * DV : nullptr;
    for (int f = tid; f < F; f += kThreads) {
        float z = Z[f];
#pragma unroll
        for (int i = 0; i < kTMax; ++i)
            if (i < T) yz[i] = fmaf(pq[f * Tp + i], z, yz[i]);
        if (GZ) {
#pragma unroll
            for (int j = 0; j < kTMax; ++j)
                if (j < T) z += pk[f * Tp + j];
            GZ[f] = z;
        }
    }
    if (state_out) {  // padding of the state stays zero
        for (int64_t e = (int64_t)F * (DV + 1) + tid; e < stride; e += kThreads) state_out[(int64_t)bh * stride + e] = 0.f;
    }

    // reductions over rows: lanes sharing a column group sit DV4 apart in a warp
#pragma unroll
    for (int i = 0; i < kTMax; ++i) {
        if (i < T) {
#pragma unroll
            for (int o = DV4; o < 32; o <<= 1) {
                y[i].x += __shfl_xor_sync(0xffffffffu, y[i].x, o);
                y[i].y += __shfl_xor_sync(0xffffffffu, y[i].y, o);
                y[i].z += __shfl_xor_sync(0xffffffffu, y[i].z, o);
                y[i].w += __shfl_xor_sync(0xffffffffu, y[i].w, o);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) yz[i] += __shfl_xor_sync(0xffffffffu, yz[i], o);
            if (lane < DV4) red[(warp * T + i) * DV4 + lane] = y[i];
            if (lane == 0) zr[warp * T + i] = yz[i];
        }
    }
    __syncthreads();
    for (int e = tid; e < T * DV; e += kThreads) {
        const int i = e / DV, c = e % DV;
        float acc = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float4 t4 = red[(w * T + i) * DV4 + (c >> 2)];
            acc += (c & 3) == 0 ? t4.x : (c & 3) == 1 ? t4.y : (c & 3) == 2 ? t4.z : t4.w;
            den += zr[w * T + i];
        }
        for (int j = 0; j <= i; ++j) {
            const float w = P[i * kTMax + j];
            acc = fmaf(w, vv[j * DV + c], acc);
            den += w;
        }
        out[(tok0 + i) * DV + c] = acc / den;
    }
}

template <typename Tin, int DV4>
cudaError_t launch_multi(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* state_out, float* out,
                         int BH, int T, int d, int n, float tau, int F, int64_t stride, uint32_t bytes, size_t dyn,
                         unsigned int* err, cudaStream_t stream) {
    auto fn = decode_multi_kernel<Tin, DV4>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t set_err[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        set_err[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDyn);
    });
    if (set_err[dev] != cudaSuccess) return set_err[dev];
    TA_TIMED(stream, "decode_multi_kernel",
             fn<<<BH, kThreads, dyn, stream>>>(q, k, v, state_in, state_out, out, T, d, n, tau, F, stride, bytes, err));
    return cudaGetLastError();
}

}  // namespace

template <typename Tin>
cudaError_t launch_decode_multi(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* state_out,
                                float* out, int BH, int T, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                                cudaStream_t stream) {
    if (T < 1 || T > kTMax || F > 1024) return cudaErrorNotSupported;
    if (dv != 16 && dv != 32 && dv != 64 && dv != 128) return cudaErrorNotSupported;
    const int64_t used_bytes = F * (dv + 1) * 4;
    const uint32_t bytes = (uint32_t)((used_bytes + 15) / 16 * 16);
    const size_t dyn = multi_layout(T, d, dv, (int)F, bytes).bytes;
    if (dyn > kMaxDyn) return cudaErrorNotSupported;
    unsigned int* err = device_error_word();
    if (!err) return cudaErrorNotSupported;
    switch (dv) {
        case 16: return launch_multi<Tin, 4>(q, k, v, state_in, state_out, out, BH, T, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
        case 32: return launch_multi<Tin, 8>(q, k, v, state_in, state_out, out, BH, T, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
        case 64: return launch_multi<Tin, 16>(q, k, v, state_in, state_out, out, BH, T, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
        default: return launch_multi<Tin, 32>(q, k, v, state_in, state_out, out, BH, T, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
    }
}

template cudaError_t launch_decode_multi<float>(const float*, const float*, const float*, const float*, float*, float*,
                                                int, int, int, int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_decode_multi<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                        const __nv_bfloat16*, const float*, float*, float*, int, int,
                                                        int, int, int, float, int64_t, int64_t, cudaStream_t);

}  // namespace ta
