// Constant-cost decode step (arXiv 2610.20637, abstract: per-token decoding
// latency is constant in N).  Per (b, h): S += phi(k) [v | 1]^T, then
// y = (c (.) phi(q))^T S and o = y[0:d_v] / y[d_v].
//
// The step is bound by HBM: each head's fp32 state (F*(d_v+1) floats) is read
// once and written once.  One CTA per head.
//
// Main path (d_v in {16, 32, 64, 128}, state <= 110 KB, F <= 1024): at entry
// one thread issues bulk (TMA) copies of the head's state into shared memory,
// completing on an mbarrier, while every thread loads the new token and its
// feature descriptors, so the three latencies overlap.  After phi(q), phi(k)
// are evaluated and the state has landed, each thread updates the rows it
// owns (one 16-byte column group per row, 128-bit shared loads) and writes
// them straight back to HBM with 128-bit stores that nothing waits for.  No
// state element stays in registers for longer than one update, so occupancy
// is set by shared memory (5 CTAs per SM at d_k 16, d_v 64, n 3).  The
// read-out sum over rows is a warp-shuffle plus shared-memory reduction.
//
// Fallback path (other d_v or larger states): the same arithmetic with
// register-staged 128-bit loads and stores, one feature tile at a time.
#include <mutex>

#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "phase.cuh"
#include "ptx.cuh"

namespace ta {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr uint32_t kWaitPolls = 1u << 22;  // bound on mbarrier polls (seconds of wall time)
constexpr int kTmaMaxBytes = 110 * 1024;
#ifndef TA_DECODE_THREADS
#define TA_DECODE_THREADS 256
#endif
constexpr int kDecThreads = TA_DECODE_THREADS;   // threads of the main decode kernel
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kTmaMaxFeatures = 1024;
constexpr int kDescPerThread = (kTmaMaxFeatures + kDecThreads - 1) / kDecThreads;
#ifndef TA_DECODE_LOAD_PIECES
#define TA_DECODE_LOAD_PIECES 1
#endif
constexpr int kLoadPieces = TA_DECODE_LOAD_PIECES;     // bulk copies per state load
constexpr int kMaxDevices = 64;

template <typename Tin, int DV4>
__global__ void __launch_bounds__(kDecThreads, kDecThreads == 256 ? 5 : 4)
decode_tma_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                  float* __restrict__ state, float* __restrict__ out, int d, int n, float tau, int F,
                  int64_t stride, uint32_t bytes, unsigned int* __restrict__ err) {
    constexpr int DV = DV4 * 4;
    constexpr int RS = kDecThreads / DV4;  // row sets
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ float xq[kMaxDk], xk[kMaxDk], vv[DV], qc[kMaxN];
    __shared__ float4 red[kDecWarps][DV4];
    __shared__ float zr[kDecWarps];
    __shared__ __align__(8) uint64_t bar;

    float* S = reinterpret_cast<float*>(dsm);
    const uint32_t soff = (bytes + 127u) & ~127u;
    float* pk = reinterpret_cast<float*>(dsm + soff);
    float* pq = pk + ((F + 3) & ~3);

    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    float* gS = state + (int64_t)bh * stride;
    TA_PHASE(3, 0, tid == 0);

    // Everything this head needs is requested at once: the state (bulk copy,
    // one thread), the new token and this thread's feature descriptors
    // (plain loads), so their latencies overlap instead of adding up.
    if (tid == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        ptx::mbar_arrive_expect_tx(&bar, bytes);
        const uint32_t piece = ((bytes + kLoadPieces - 1) / kLoadPieces + 15u) & ~15u;
        for (uint32_t o = 0; o < bytes; o += piece) {
            const uint32_t sz = bytes - o < piece ? bytes - o : piece;
            ptx::bulk_g2s(reinterpret_cast<unsigned char*>(S) + o, reinterpret_cast<const unsigned char*>(gS) + o, sz,
                          &bar);
        }
    }
    const PackedFeat* tab = feat_table(d, n);
    PackedFeat pf[kDescPerThread];
#pragma unroll
    for (int j = 0; j < kDescPerThread; ++j) {
        const int f = tid + j * kDecThreads;
        if (tab && f < F) pf[j] = tab[f];
    }
    float aq = 0.f, ak = 0.f, av = 0.f;
    if (tid < d) {
        aq = ldf(q + (int64_t)bh * d + tid);
        ak = ldf(k + (int64_t)bh * d + tid);
    }
    if (tid < DV) av = ldf(v + (int64_t)bh * DV + tid);
    if (tid < d) {
        xq[tid] = aq;
        xk[tid] = ak;
    }
    if (tid < DV) vv[tid] = av;
    if (tid < n) qc[tid] = query_coeff(tid, tau);
    TA_PHASE(3, 1, tid == 0);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kDescPerThread; ++j) {
        const int f = tid + j * kDecThreads;
        if (f < F) {
            const FeatDesc dk = tab ? desc_from_packed(pf[j], qc, false) : make_desc(d, n, f, tau, false);
            const FeatDesc dq = tab ? desc_from_packed(pf[j], qc, true) : make_desc(d, n, f, tau, true);
            pk[f] = eval_desc(dk, xk);
            pq[f] = eval_desc(dq, xq);
        }
    }
    TA_PHASE(3, 2, tid == 0);
    // every thread observes the copy's completion itself; the block agrees
    // on the outcome so that a timeout leaves as one
    const bool landed = ptx::mbar_wait(&bar, 0, kWaitPolls);
    TA_PHASE(3, 7, tid == 0);
    if (!__syncthreads_and(landed)) {
        if (tid == 0) atomicOr(err, kErrDecodeLoad);
        if (!landed) ptx::mbar_wait(&bar, 0, kWaitPolls);  // one more bound for the copy in flight
        return;
    }

    TA_PHASE(3, 3, tid == 0);
    // each updated row leaves straight from registers: a warp stores 512
    // contiguous bytes per instruction, and nothing waits for the stores
    const int cg = tid % DV4, rs = tid / DV4;
    const float4 v4 = reinterpret_cast<const float4*>(vv)[cg];
    const float4* S4 = reinterpret_cast<const float4*>(S);
    float4* G4 = reinterpret_cast<float4*>(gS);
    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int r = rs; r < F; r += RS) {
        const float a = pk[r], b = pq[r];
        float4 s = S4[r * DV4 + cg];
        s.x = fmaf(a, v4.x, s.x);
        s.y = fmaf(a, v4.y, s.y);
        s.z = fmaf(a, v4.z, s.z);
        s.w = fmaf(a, v4.w, s.w);
        G4[r * DV4 + cg] = s;
        y.x = fmaf(b, s.x, y.x);
        y.y = fmaf(b, s.y, y.y);
        y.z = fmaf(b, s.z, y.z);
        y.w = fmaf(b, s.w, y.w);
    }
    float yz = 0.f;
    const float* Z = S + F * DV;
    float* GZ = gS + (int64_t)F * DV;
    for (int f = tid; f < F; f += kDecThreads) {
        const float z = Z[f] + pk[f];
        GZ[f] = z;
        yz = fmaf(pq[f], z, yz);
    }
    TA_PHASE(3, 4, tid == 0);

    // read-out: lanes sharing a column group sit DV4 apart inside a warp
#pragma unroll
    for (int o = DV4; o < 32; o <<= 1) {
        y.x += __shfl_xor_sync(0xffffffffu, y.x, o);
        y.y += __shfl_xor_sync(0xffffffffu, y.y, o);
        y.z += __shfl_xor_sync(0xffffffffu, y.z, o);
        y.w += __shfl_xor_sync(0xffffffffu, y.w, o);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) yz += __shfl_xor_sync(0xffffffffu, yz, o);
    const int warp = tid >> 5, lane = tid & 31;
    if (lane < DV4) red[warp][lane] = y;
    if (lane == 0) zr[warp] = yz;
    __syncthreads();
    if (tid < DV) {
        const int g = tid >> 2, c = tid & 3;
        float acc = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
            const float4 t = red[w][g];
            acc += c == 0 ? t.x : c == 1 ? t.y : c == 2 ? t.z : t.w;
            den += zr[w];
        }
        out[(int64_t)bh * DV + tid] = acc / den;
    }
    TA_PHASE(3, 5, tid == 0);
    TA_PHASE(3, 6, tid == 0);
}

constexpr int kFeatTile = 1024;  // features whose phi(q), phi(k) sit in smem at once
constexpr int kRows = 10;        // S_v rows per thread held in registers per batch

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
decode_generic_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                      float* __restrict__ state, float* __restrict__ out, int d, int dv, int n,
                      float tau, int F, int64_t stride) {
    __shared__ float xs_q[kMaxDk], xs_k[kMaxDk], vs[kMaxDv], qc[kMaxN];
    __shared__ float pk[kFeatTile], pq[kFeatTile];
    __shared__ float4 red[kThreads];
    __shared__ float zred[kWarps];

    const int bh = blockIdx.x;
    const int tid = threadIdx.x;
    const int dv4 = dv >> 2;
    const int rsets = kThreads / dv4;
    const int cg = tid % dv4;
    const int rs = tid / dv4;
    const bool active = rs < rsets;

    float* Sv = state + (int64_t)bh * stride;
    float* Z = Sv + (int64_t)F * dv;
    const PackedFeat* tab = feat_table(d, n);

    for (int i = tid; i < d; i += kThreads) {
        xs_q[i] = ldf(q + (int64_t)bh * d + i);
        xs_k[i] = ldf(k + (int64_t)bh * d + i);
    }
    for (int i = tid; i < dv; i += kThreads) vs[i] = ldf(v + (int64_t)bh * dv + i);
    if (tid < n) qc[tid] = query_coeff(tid, tau);

    float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
    float yz = 0.f;

    for (int fb = 0; fb < F; fb += kFeatTile) {
        const int fe = min(F, fb + kFeatTile);
        __syncthreads();  // inputs ready; previous tile's pk/pq consumed
        for (int f = fb + tid; f < fe; f += kThreads) {
            pk[f - fb] = eval_desc(get_desc(tab, d, n, f, tau, qc, false), xs_k);
            pq[f - fb] = eval_desc(get_desc(tab, d, n, f, tau, qc, true), xs_q);
        }
        __syncthreads();
        const float4 v4 = active ? *reinterpret_cast<const float4*>(vs + cg * 4) : make_float4(0, 0, 0, 0);
        for (int r0 = fb + rs; r0 < fe; r0 += kRows * rsets) {
            float4 s[kRows];
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                const int r = r0 + i * rsets;
                if (active && r < fe) s[i] = *reinterpret_cast<const float4*>(Sv + (int64_t)r * dv + cg * 4);
            }
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
        }
        for (int f = fb + tid; f < fe; f += kThreads) {
            const float z = Z[f] + pk[f - fb];
            Z[f] = z;
            yz = fmaf(pq[f - fb], z, yz);
        }
    }

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
        for (int w = 0; w < kWarps; ++w) den += zred[w];
        out[(int64_t)bh * dv + tid] = acc / den;
    }
}

template <typename Tin, int DV4>
cudaError_t launch_tma(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH, int d,
                       int n, float tau, int F, int64_t stride, uint32_t bytes, size_t dyn,
                       unsigned int* err, cudaStream_t stream) {
    auto fn = decode_tma_kernel<Tin, DV4>;
    if (dyn > 48 * 1024) {
        static std::once_flag once[kMaxDevices];
        static cudaError_t set_err[kMaxDevices];
        int dev = 0;
        cudaGetDevice(&dev);
        if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
        std::call_once(once[dev], [&]() {
            set_err[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, kTmaMaxBytes + 8192);
        });
        if (set_err[dev] != cudaSuccess) return set_err[dev];
    }
    TA_TIMED(stream, "decode_tma_kernel",
             fn<<<BH, kDecThreads, dyn, stream>>>(q, k, v, state, out, d, n, tau, F, stride, bytes, err));
    return cudaGetLastError();
}

}  // namespace

template <typename Tin>
cudaError_t launch_decode(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH,
                          int d, int dv, int n, float tau, int64_t F, int64_t stride, cudaStream_t stream) {
    if (BH == 0) return cudaSuccess;
    const int64_t used_bytes = F * (dv + 1) * 4;
    const uint32_t bytes = (uint32_t)((used_bytes + 15) / 16 * 16);
    const size_t dyn = ((bytes + 127u) & ~127u) + 2 * (size_t)((F + 3) & ~3) * 4;
    unsigned int* err = device_error_word();
    const bool tma_ok = err != nullptr && used_bytes <= kTmaMaxBytes && dyn <= (size_t)kTmaMaxBytes + 8192 &&
                        F <= kTmaMaxFeatures;
    if (err != nullptr) {  // many heads of a small state: the persistent warp-specialised kernel
        const cudaError_t e = launch_decode_ws(q, k, v, state, out, BH, d, dv, n, tau, F, stride, stream);
        if (e != cudaErrorNotSupported) return e;
    }
    if (tma_ok) {
        switch (dv) {
            case 16: return launch_tma<Tin, 4>(q, k, v, state, out, BH, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
            case 32: return launch_tma<Tin, 8>(q, k, v, state, out, BH, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
            case 64: return launch_tma<Tin, 16>(q, k, v, state, out, BH, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
            case 128: return launch_tma<Tin, 32>(q, k, v, state, out, BH, d, n, tau, (int)F, stride, bytes, dyn, err, stream);
            default: break;
        }
    }
    TA_TIMED(stream, "decode_generic_kernel",
             decode_generic_kernel<Tin><<<BH, kThreads, 0, stream>>>(q, k, v, state, out, d, dv, n, tau,
                                                                     (int)F, stride));
    return cudaGetLastError();
}

template cudaError_t launch_decode<float>(const float*, const float*, const float*, float*, float*, int, int,
                                          int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_decode<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                  const __nv_bfloat16*, float*, float*, int, int, int, int,
                                                  float, int64_t, int64_t, cudaStream_t);

}  // namespace ta
