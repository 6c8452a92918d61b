// Persistent, warp-specialised decode step for d_v = 64 and states of at most
// 256 features (the decode workload: d_k 16, n 3, 153 x 65 floats per head).
// Same arithmetic as the one-CTA-per-head kernel in decode.cu (the paper's
// constant-cost decode, arXiv 2610.20637, abstract):
//   S += phi(k) [v | 1]^T,  y = (c (.) phi(q))^T S,  o = y[0:64] / y[64].
//
// One CTA per SM walks the heads blockIdx.x, blockIdx.x + gridDim.x, ...
// One producer thread keeps a ring of state buffers in shared memory full:
// for each head a bulk copy of its state and of its new token (q, k, v)
// completing on the buffer's mbarrier, issued as soon as the buffer is free
// (the first copies before anything else in the kernel), so several heads'
// loads per SM are always in flight.  Four consumer warpgroups take the heads
// in turn; a warpgroup evaluates phi(k), phi(q) for its head, updates the rows
// (one 16-byte column group per thread per row, stored straight to HBM),
// reduces the read-out and writes o, synchronising only its own 128 threads
// (named barriers), then hands the buffer back.
//
// The ring holds a multiple of four buffers, so head i's buffer (i mod the
// ring size) is only ever consumed by warpgroup i mod 4, in order: no
// warpgroup can wait on a buffer phase while an earlier phase of the same
// buffer is still outstanding, which a parity wait could not tell apart.
//
// With at most 256 features the series has degree <= 2 for every supported
// d_k (d_k 16: n <= 3; d_k 32, 64: n <= 2), so each thread derives its
// features' indices and weights arithmetically once, with no table lookup
// in front of the first copies.
#include <mutex>

#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace ta {

namespace {

constexpr int kDV = 64, kDV4 = 16;
constexpr int kWG = 4;                      // consumer warpgroups
constexpr int kWGThreads = 128;
constexpr int kThreadsWS = kWG * kWGThreads + 32;
constexpr int kMaxF = 256;
constexpr int kMaxBuf = 8;  // a multiple of kWG
constexpr uint32_t kWaitPolls = 1u << 22;
constexpr size_t kMaxDynWS = 218 * 1024;  // with the static arrays, within the 227 KB per CTA
constexpr int kMaxDevices = 64;

struct WGArea {                 // per consumer warpgroup
    float pk[kMaxF], pq[kMaxF];
    float4 red[3][4][kDV4];     // column partials per degree (one degree for the Taylor read-out)
    float zr[3][4];
    int fail;                   // written only before a warpgroup barrier, read after it
};

__device__ __forceinline__ void wg_sync(int wg) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + wg), "r"(kWGThreads) : "memory");
}

// CENTRED: the read-out of the mean-centred softmax expansion (order 1 or 2)
// over the n = 3 state instead of the Taylor read-out: the query features
// carry no tau^m/m!, the row walk keeps one accumulator per degree, and the
// epilogue combines the three per-degree read-outs R_m (Su Jianlin, "Taylor
// expansions of logsumexp and softmax", kexue.fm translation 11814, sections
// "Calculating the Gradient" and "Linear Attention"):
//   n = R_0[z], V = R_0[v], qkbar = R_1[z] / n,
//   o = V/n + tau (R_1[v] - qkbar V)/n
//     [+ (tau^2 (R_2[v] - 2 qkbar R_1[v] + qkbar^2 V) - tau^2 (R_2[z] - n qkbar^2) V/n) / (2n)].
template <typename Tin, bool CENTRED>
__global__ void __launch_bounds__(kThreadsWS, 1)
decode_ws_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 float* __restrict__ state, float* __restrict__ out, int BH, int d, int n, float tau, int F,
                 int64_t stride, uint32_t bytes, uint32_t buf_bytes, int nbuf, int order,
                 unsigned int* __restrict__ err) {
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ __align__(8) uint64_t full[kMaxBuf], empty[kMaxBuf];
    __shared__ int s_bad;
    WGArea* wga = reinterpret_cast<WGArea*>(dsm + (size_t)nbuf * buf_bytes);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nheads = BH > (int)blockIdx.x ? (BH - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const uint32_t tok_in = (uint32_t)(d * sizeof(Tin)), tok_v = (uint32_t)(kDV * sizeof(Tin));
    // token area of a buffer: q, k, v rows right after the state, 16-byte aligned
    const uint32_t offq = (bytes + 15u) & ~15u, offk = offq + ((tok_in + 15u) & ~15u),
                   offv = offk + ((tok_in + 15u) & ~15u);
    const int producer = kWG * kWGThreads;
    auto issue = [&](int i) {
        const int b = i % nbuf;
        const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
        unsigned char* buf = dsm + (size_t)b * buf_bytes;
        ptx::mbar_arrive_expect_tx(&full[b], bytes + 2 * tok_in + tok_v);
        ptx::bulk_g2s(buf, state + h * stride, bytes, &full[b]);
        ptx::bulk_g2s(buf + offq, q + h * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + offk, k + h * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + offv, v + h * kDV, tok_v, &full[b]);
    };

    // launched with programmatic dependent launch: the next grid in the
    // stream may be scheduled now, and this grid's first memory access (the
    // producer's first copy; every other access follows one of its copies)
    // waits until the previous grid has completed and its writes are visible
    ptx::pdl_launch_dependents();
    // the producer sets up the ring and starts the first copies at once
    int issued = 0;
    if (tid == producer) {
        for (int i = 0; i < nbuf; ++i) {
            ptx::mbar_init(&full[i], 1);
            ptx::mbar_init(&empty[i], 1);
        }
        ptx::fence_mbar_init();
        ptx::pdl_wait_primary();
        for (; issued < nbuf && issued < nheads; ++issued) issue(issued);
    }
    if (tid == 0) s_bad = 0;
    if (tid < kWG) wga[tid].fail = 0;
    __syncthreads();

    if (warp == kWG * kWGThreads / 32) {
        if (lane == 0) {
            int i = issued;
            for (; i < nheads; ++i) {
                const int b = i % nbuf;
                if (!ptx::mbar_wait_or_abort(&empty[b], ((i / nbuf) - 1) & 1, kWaitPolls, &s_bad)) break;
                issue(i);
            }
            // copies that no warpgroup consumed (only after a failure) land before the CTA leaves
            for (int j = (i > nbuf ? i - nbuf : 0); j < i; ++j)
                ptx::mbar_wait(&full[j % nbuf], (j / nbuf) & 1, kWaitPolls);
        }
    } else {
        const int wg = warp >> 2, t = tid & (kWGThreads - 1), wl = (warp & 3);
        WGArea& A = wga[wg];
        const int cg = t % kDV4, rs = t / kDV4;  // 8 row sets
        // this thread's features t and t + 128: phi_f(x) = w x_i x_j (factors
        // past the degree are 1); the query weight carries tau^m / m!
        int m0, i0, j0, m1, i1, j1;
        float w0, w1;
        feature_deg2(d, t < F ? t : 0, m0, i0, j0, w0);
        feature_deg2(d, t + kWGThreads < F ? t + kWGThreads : 0, m1, i1, j1, w1);
        const float wq0 = CENTRED ? w0 : w0 * query_coeff(m0, tau), wq1 = CENTRED ? w1 : w1 * query_coeff(m1, tau);
        for (int i = wg; i < nheads; i += kWG) {
            const int b = i % nbuf;  // == wg modulo kWG: only this warpgroup consumes buffer b
            if (!ptx::mbar_wait_or_abort(&full[b], (i / nbuf) & 1, kWaitPolls, &s_bad)) A.fail = 1;
            wg_sync(wg);
            if (A.fail) break;  // the same value for all 128 threads: set only before this barrier
            const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
            const unsigned char* buf = dsm + (size_t)b * buf_bytes;
            const Tin* xq = reinterpret_cast<const Tin*>(buf + offq);
            const Tin* xk = reinterpret_cast<const Tin*>(buf + offk);
            const Tin* vv = reinterpret_cast<const Tin*>(buf + offv);
            if (t < F) {
                const float ki = m0 >= 1 ? to_float(xk[i0]) : 1.0f, kj = m0 >= 2 ? to_float(xk[j0]) : 1.0f;
                const float qi = m0 >= 1 ? to_float(xq[i0]) : 1.0f, qj = m0 >= 2 ? to_float(xq[j0]) : 1.0f;
                A.pk[t] = w0 * ki * kj;
                A.pq[t] = wq0 * qi * qj;
            }
            if (t + kWGThreads < F) {
                const float ki = m1 >= 1 ? to_float(xk[i1]) : 1.0f, kj = m1 >= 2 ? to_float(xk[j1]) : 1.0f;
                const float qi = m1 >= 1 ? to_float(xq[i1]) : 1.0f, qj = m1 >= 2 ? to_float(xq[j1]) : 1.0f;
                A.pk[t + kWGThreads] = w1 * ki * kj;
                A.pq[t + kWGThreads] = wq1 * qi * qj;
            }
            const float4 v4 = make_float4(to_float(vv[4 * cg]), to_float(vv[4 * cg + 1]), to_float(vv[4 * cg + 2]),
                                          to_float(vv[4 * cg + 3]));
            wg_sync(wg);
            const float4* S4 = reinterpret_cast<const float4*>(buf);
            float4* G4 = reinterpret_cast<float4*>(state + h * stride);
            constexpr int ND = CENTRED ? 3 : 1;  // accumulators: per degree, or one
            float4 y[ND];
#pragma unroll
            for (int m = 0; m < ND; ++m) y[m] = make_float4(0.f, 0.f, 0.f, 0.f);
            // rows [lo, hi) of this thread's row set into accumulator m
            auto walk = [&](int lo, int hi, float4& acc) {
                const int r0 = lo + ((rs - lo) % (kWGThreads / kDV4) + kWGThreads / kDV4) % (kWGThreads / kDV4);
#pragma unroll 4
                for (int r = r0; r < hi; r += kWGThreads / kDV4) {
                    const float a = A.pk[r], c = A.pq[r];
                    float4 s = S4[r * kDV4 + cg];
                    s.x = fmaf(a, v4.x, s.x);
                    s.y = fmaf(a, v4.y, s.y);
                    s.z = fmaf(a, v4.z, s.z);
                    s.w = fmaf(a, v4.w, s.w);
                    G4[r * kDV4 + cg] = s;
                    acc.x = fmaf(c, s.x, acc.x);
                    acc.y = fmaf(c, s.y, acc.y);
                    acc.z = fmaf(c, s.z, acc.z);
                    acc.w = fmaf(c, s.w, acc.w);
                }
            };
            if (CENTRED) {
                walk(0, 1, y[0]);
                walk(1, d + 1, y[ND > 1 ? 1 : 0]);
                walk(d + 1, F, y[ND > 2 ? 2 : 0]);
            } else {
                walk(0, F, y[0]);
            }
            float yz[ND];
#pragma unroll
            for (int m = 0; m < ND; ++m) yz[m] = 0.f;
            const float* Z = reinterpret_cast<const float*>(buf) + (int64_t)F * kDV;
            float* GZ = state + h * stride + (int64_t)F * kDV;
            for (int f = t; f < F; f += kWGThreads) {
                const float z = Z[f] + A.pk[f];
                GZ[f] = z;
                const int m = CENTRED ? (f == 0 ? 0 : (f <= d ? 1 : 2)) : 0;
#pragma unroll
                for (int mm = 0; mm < ND; ++mm)
                    if (mm == m) yz[mm] = fmaf(A.pq[f], z, yz[mm]);
            }
            // the buffer has been read: hand it back once the whole warpgroup is past here
            ptx::fence_proxy_async_smem();
#pragma unroll
            for (int m = 0; m < ND; ++m) {
                y[m].x += __shfl_xor_sync(0xffffffffu, y[m].x, 16);
                y[m].y += __shfl_xor_sync(0xffffffffu, y[m].y, 16);
                y[m].z += __shfl_xor_sync(0xffffffffu, y[m].z, 16);
                y[m].w += __shfl_xor_sync(0xffffffffu, y[m].w, 16);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) yz[m] += __shfl_xor_sync(0xffffffffu, yz[m], o);
                if (lane < kDV4) A.red[m][wl][lane] = y[m];
                if (lane == 0) A.zr[m][wl] = yz[m];
            }
            wg_sync(wg);
            if (t == 0) ptx::mbar_arrive(&empty[b]);
            if (t < kDV) {
                const int g4 = t >> 2, c4 = t & 3;
                float R[ND], Rz[ND];
#pragma unroll
                for (int m = 0; m < ND; ++m) {
                    R[m] = 0.f;
                    Rz[m] = 0.f;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const float4 r4 = A.red[m][w][g4];
                        R[m] += c4 == 0 ? r4.x : c4 == 1 ? r4.y : c4 == 2 ? r4.z : r4.w;
                        Rz[m] += A.zr[m][w];
                    }
                }
                float o;
                if (CENTRED) {
                    const float cnt = Rz[0], V = R[0], qkbar = Rz[ND > 1 ? 1 : 0] / cnt;
                    o = V / cnt + tau * (R[ND > 1 ? 1 : 0] - qkbar * V) / cnt;
                    if (order >= 2) {
                        const float t2 = tau * tau;
                        const float sum_a2v = t2 * (R[ND > 2 ? 2 : 0] - 2.0f * qkbar * R[ND > 1 ? 1 : 0] + qkbar * qkbar * V);
                        const float sum_a2 = t2 * (Rz[ND > 2 ? 2 : 0] - cnt * qkbar * qkbar);
                        o += (sum_a2v - sum_a2 * V / cnt) / (2.0f * cnt);
                    }
                } else {
                    o = R[0] / Rz[0];
                }
                out[h * kDV + t] = o;
            }
            // A.pk, A.pq, A.red are rewritten only after the next head's first barrier
        }
    }
    __syncthreads();
    if (tid == 0 && s_bad) atomicOr(err, kErrDecodeLoad);
}

template <typename Tin, bool CENTRED>
cudaError_t launch_ws(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH, int d, int dv,
                      int n, float tau, int64_t F, int64_t stride, int order, cudaStream_t stream) {
    // features of degree <= 2 only (always the case for F <= 256 at the supported d_k)
    if (dv != kDV || F > kMaxF || n > 3 || (d * (int)sizeof(Tin)) % 16 != 0) return cudaErrorNotSupported;
    static std::once_flag once[kMaxDevices];
    static cudaError_t set_err[kMaxDevices];
    static int num_sms[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        set_err[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(decode_ws_kernel<Tin, CENTRED>),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDynWS);
        if (set_err[dev] == cudaSuccess)
            set_err[dev] = cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    if (set_err[dev] != cudaSuccess) return set_err[dev];
    if (BH < 2 * num_sms[dev]) return cudaErrorNotSupported;  // few heads: one CTA per head is as good
    const uint32_t bytes = (uint32_t)((F * (kDV + 1) * 4 + 15) / 16 * 16);
    const uint32_t tok = (uint32_t)(((d * sizeof(Tin) + 15) / 16 * 16) * 2 + kDV * sizeof(Tin));
    const uint32_t buf_bytes = (bytes + 15u) / 16u * 16u + tok;
    const uint32_t buf_al = (buf_bytes + 127u) & ~127u;
    const size_t area = kWG * sizeof(WGArea);
    // a multiple of the warpgroup count, so that every buffer has one consumer
    int nbuf = (int)((kMaxDynWS - area) / buf_al);
    if (nbuf > kMaxBuf) nbuf = kMaxBuf;
    nbuf -= nbuf % kWG;
    if (nbuf < kWG) return cudaErrorNotSupported;
    const size_t dyn = (size_t)nbuf * buf_al + area;
    unsigned int* err = device_error_word();
    if (!err) return cudaErrorNotSupported;
    const int grid = num_sms[dev] < BH ? num_sms[dev] : BH;
    cudaError_t e = cudaSuccess;
    TA_TIMED(stream, CENTRED ? "centred_decode_ws_kernel" : "decode_ws_kernel",
             e = launch_maybe_pdl(decode_ws_kernel<Tin, CENTRED>, dim3(grid), dim3(kThreadsWS), dyn, stream, true, q,
                                  k, v, state, out, BH, d, n, tau, (int)F, stride, bytes, buf_al, nbuf, order, err));
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

template <typename Tin>
cudaError_t launch_decode_ws(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH, int d,
                             int dv, int n, float tau, int64_t F, int64_t stride, cudaStream_t stream) {
    return launch_ws<Tin, false>(q, k, v, state, out, BH, d, dv, n, tau, F, stride, 0, stream);
}

template <typename Tin>
cudaError_t launch_centred_decode_ws(const Tin* q, const Tin* k, const Tin* v, float* state, float* out, int BH,
                                     int d, int dv, int order, float tau, int64_t F, int64_t stride,
                                     cudaStream_t stream) {
    return launch_ws<Tin, true>(q, k, v, state, out, BH, d, dv, 3, tau, F, stride, order, stream);
}

template cudaError_t launch_centred_decode_ws<float>(const float*, const float*, const float*, float*, float*, int,
                                                     int, int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_centred_decode_ws<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                             const __nv_bfloat16*, float*, float*, int, int, int, int,
                                                             float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_decode_ws<float>(const float*, const float*, const float*, float*, float*, int, int, int,
                                             int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_decode_ws<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                     const __nv_bfloat16*, float*, float*, int, int, int, int, float,
                                                     int64_t, int64_t, cudaStream_t);

}  // namespace ta
