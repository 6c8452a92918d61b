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
#include <type_traits>

#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "phase.cuh"
#include "ptx.cuh"

namespace ta {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTMax = 16;
constexpr uint32_t kWaitPolls = 1u << 22;
constexpr size_t kMaxDyn = 226 * 1024;  // the 227 KB per-block limit, less static shared memory
constexpr int kMaxDevices = 64;
constexpr int kTcMinTokens = 8;  // the tensor-core multi-token kernel takes T > 8

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

// ---------------------------------------------------------------- persistent form
// The same step for d_v = 64 and features of degree <= 2 (F <= 256), many
// heads: one CTA per SM walks the heads blockIdx.x, blockIdx.x + gridDim.x,
// ...  Two warpgroups take the heads in turn, each with its own ring buffer
// (the head's state and its T tokens' q, k, v rows, brought in by bulk
// copies that complete on the buffer's mbarrier): warpgroup g takes heads g,
// g + 2, ... of the CTA and, once it has read a head's buffer, itself issues
// the copies of its next head into it, so a copy is in flight while it
// finishes the head before.  A warpgroup evaluates phi(k_j), phi(q_j) and
// the block's pairwise weights into its own area, walks the state rows once
// (read-out of all T tokens from the old row, the T rank-one updates, the new
// row stored straight to HBM), hands the buffer on, then reduces the
// read-out and writes the outputs.  In the walk each thread keeps its column
// group of the T v rows in registers, so a row costs one state load and the
// row's read-out and update coefficients (broadcast within the row set) from
// shared memory; two warpgroups and no other warp leave room for about 250
// registers a thread.
constexpr int kWGm = 2;
constexpr int kWGmThreads = 128;
constexpr int kThreadsWSm = kWGm * kWGmThreads;
constexpr int kDVw = 64, kDV4w = 16;
constexpr size_t kMaxDynWSm = 226 * 1024;

struct MultiWsLayout {
    uint32_t offq, offk, offv, buf;                  // one ring buffer: state, then the q, k, v rows
    uint32_t pk, pq, vf, p, zr, xq, xk, area;        // one warpgroup area
    uint32_t desc, bytes;                            // the feature table after the areas; the total
};

// Features per warpgroup walk; the q, k rows held as fp32 with one extra
// slot of 1 (stride d + 1) so that degree 0 and 1 features read it as their
// missing factors.
__host__ __device__ inline MultiWsLayout multi_ws_layout(int T, int d, int F, uint32_t state_bytes, uint32_t esize) {
    auto al = [](uint32_t x) { return (x + 127u) & ~127u; };
    MultiWsLayout L;
    const uint32_t Tp = (uint32_t)((T + 3) & ~3);
    L.offq = al(state_bytes);
    L.offk = L.offq + al((uint32_t)(T * d) * esize);
    L.offv = L.offk + al((uint32_t)(T * d) * esize);
    L.buf = L.offv + al((uint32_t)(T * kDVw) * esize);
    // pk, pq [F][Tp]; after the row walk the same space holds the column
    // partials [8 row sets][T][64]
    const uint32_t coeff = al((uint32_t)F * Tp * 4);
    const uint32_t partials = al((uint32_t)(8 * T * kDVw) * 4);
    L.pk = 0;
    L.pq = coeff;
    const uint32_t span = 2 * coeff > partials ? 2 * coeff : partials;
    L.vf = span;                                   // v rows as fp32 [T][64]
    L.p = L.vf + al((uint32_t)(T * kDVw) * 4);    // pairwise weights [16][16]
    L.zr = L.p + al((uint32_t)(kTMax * kTMax) * 4);  // normaliser partials [8][16]
    L.xq = L.zr + al((uint32_t)(8 * kTMax) * 4);
    L.xk = L.xq + al((uint32_t)(T * (d + 1)) * 4);
    L.area = L.xk + al((uint32_t)(T * (d + 1)) * 4);
    L.desc = kWGm * (L.buf + L.area);              // [F] float4: {a | c << 8, w, w tau^m/m!, 0}
    L.bytes = L.desc + al((uint32_t)F * 16);
    return L;
}

__device__ __forceinline__ void wgm_sync(int wg) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + wg), "r"(kWGmThreads) : "memory");
}

template <typename Tin>
__global__ void __launch_bounds__(kThreadsWSm, 1)
decode_multi_ws_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                       const float* state_in, float* state_out, float* __restrict__ out, int BH, int T, int d, int n,
                       float tau, int F, int64_t stride, uint32_t bytes, unsigned int* __restrict__ err) {
    extern __shared__ __align__(128) unsigned char dsm[];
    __shared__ __align__(8) uint64_t full[kWGm];
    __shared__ int s_bad, s_fail[kWGm];
    const MultiWsLayout L = multi_ws_layout(T, d, F, bytes, (uint32_t)sizeof(Tin));
    unsigned char* areas = dsm + (size_t)kWGm * L.buf;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int nheads = BH > (int)blockIdx.x ? (BH - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const uint32_t tok_in = (uint32_t)(T * d) * (uint32_t)sizeof(Tin), tok_v = (uint32_t)(T * kDVw) * (uint32_t)sizeof(Tin);
    auto issue = [&](int i) {  // head i of this CTA into buffer i mod 2
        const int b = i % kWGm;
        const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
        unsigned char* buf = dsm + (size_t)b * L.buf;
        ptx::mbar_arrive_expect_tx(&full[b], bytes + 2 * tok_in + tok_v);
        ptx::bulk_g2s(buf, state_in + h * stride, bytes, &full[b]);
        ptx::bulk_g2s(buf + L.offq, q + h * T * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + L.offk, k + h * T * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + L.offv, v + h * T * kDVw, tok_v, &full[b]);
    };

    // launched with programmatic dependent launch: every memory access of the
    // grid follows thread 0's wait on the previous grid (directly, or through
    // the barrier below)
    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < kWGm; ++i) ptx::mbar_init(&full[i], 1);
        ptx::fence_mbar_init();
        ptx::pdl_wait_primary();
        for (int i = 0; i < kWGm && i < nheads; ++i) issue(i);
        s_bad = 0;
    }
    if (tid < kWGm) s_fail[tid] = 0;
    // the feature table: degree, indices (d for a missing factor, which
    // reads the slot of 1 after each q, k row) and both weights
    float4* desc = reinterpret_cast<float4*>(dsm + L.desc);
    for (int f = tid; f < F; f += kThreadsWSm) {
        int m, a, c2;
        float w;
        feature_deg2(d, f, m, a, c2, w);
        if (m < 2) c2 = d;
        if (m < 1) a = d;
        desc[f] = make_float4(__int_as_float(a | (c2 << 8)), w, w * query_coeff(m, tau), 0.f);
    }
    __syncthreads();

    {
        const int wg = warp >> 2, t = tid & (kWGmThreads - 1);
        unsigned char* area = areas + (size_t)wg * L.area;
        float* pk = reinterpret_cast<float*>(area + L.pk);
        float* pq = reinterpret_cast<float*>(area + L.pq);
        float* red = reinterpret_cast<float*>(area + L.pk);  // after the row walk
        float* vf = reinterpret_cast<float*>(area + L.vf);
        float* P = reinterpret_cast<float*>(area + L.p);
        float* zr = reinterpret_cast<float*>(area + L.zr);
        float* qf = reinterpret_cast<float*>(area + L.xq);
        float* kf = reinterpret_cast<float*>(area + L.xk);
        const int Tp = (T + 3) & ~3, Tp4 = Tp / 4;
        const int zi = t & 15, zs = t >> 4;  // the z column: token zi, row set zs
        const int cg = t % kDV4w, rs = t / kDV4w;  // 8 row sets
        TA_PHASE_VARS(p_t, p_wait = 0, p_prep = 0, p_walk = 0, p_z = 0, p_red = 0, p_out = 0);
        for (int i = wg; i < nheads; i += kWGm) {
            const int b = i % kWGm;  // == wg: only this warpgroup consumes buffer b
            TA_PHASE_T0(p_t);
            if (!ptx::mbar_wait_or_abort(&full[b], (i / kWGm) & 1, kWaitPolls, &s_bad)) s_fail[wg] = 1;
            wgm_sync(wg);
            TA_PHASE_ACC(p_wait, p_t);
            TA_PHASE_T0(p_t);
            if (s_fail[wg]) {  // the same value for all 128 threads: set only before this barrier
                // the copies may still land: wait for them (bounded) before the block can exit
                if (t == 0) ptx::mbar_wait(&full[b], (i / kWGm) & 1, kWaitPolls);
                break;
            }
            const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
            const unsigned char* buf = dsm + (size_t)b * L.buf;
            const Tin* xq = reinterpret_cast<const Tin*>(buf + L.offq);
            const Tin* xk = reinterpret_cast<const Tin*>(buf + L.offk);
            const Tin* xv = reinterpret_cast<const Tin*>(buf + L.offv);
            // q, k rows to fp32 with the slot of 1; v rows to fp32
            for (int e = t; e < T * (d + 1); e += kWGmThreads) {
                const int j = e / (d + 1), c = e - j * (d + 1);
                qf[e] = c < d ? to_float(xq[j * d + c]) : 1.f;
                kf[e] = c < d ? to_float(xk[j * d + c]) : 1.f;
            }
            for (int e = t; e < T * kDVw; e += kWGmThreads) vf[e] = to_float(xv[e]);
            wgm_sync(wg);
            // phi(k_j) and (tau^m/m!) phi(q_j), feature-major with the tokens
            // contiguous; one thread per feature and four tokens
            for (int u = t; u < F * Tp4; u += kWGmThreads) {
                const int f = Tp4 == 4 ? u >> 2 : Tp4 == 2 ? u >> 1 : Tp4 == 1 ? u : u / 3;
                const int j0 = 4 * (u - f * Tp4);
                const float4 fd = desc[f];
                const int a = __float_as_int(fd.x) & 255, c2 = __float_as_int(fd.x) >> 8;
                float kk[4], qq[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    const int j = j0 + jj < T ? j0 + jj : 0;  // padded tokens get coefficient 0 below
                    const float* kr = kf + j * (d + 1);
                    const float* qr = qf + j * (d + 1);
                    const float live = j0 + jj < T ? 1.f : 0.f;
                    kk[jj] = live * fd.y * kr[a] * kr[c2];
                    qq[jj] = live * fd.z * qr[a] * qr[c2];
                }
                reinterpret_cast<float4*>(pk)[u] = make_float4(kk[0], kk[1], kk[2], kk[3]);
                reinterpret_cast<float4*>(pq)[u] = make_float4(qq[0], qq[1], qq[2], qq[3]);
            }
            // the block's own causal part: K(tau q_i.k_j) for j <= i
            for (int e = t; e < kTMax * kTMax; e += kWGmThreads) {
                const int ii = e / kTMax, j = e % kTMax;
                float w = 0.f;
                if (ii < T && j <= ii) {
                    float dot = 0.f;
                    for (int c = 0; c < d; ++c) dot = fmaf(qf[ii * (d + 1) + c], kf[j * (d + 1) + c], dot);
                    w = taylor_kernel(tau * dot, n);
                }
                P[e] = w;
            }
            wgm_sync(wg);
            TA_PHASE_ACC(p_prep, p_t);
            TA_PHASE_T0(p_t);

            // one walk over the state rows: read-out of every token from the
            // old row, then the T rank-one updates, the new row to HBM
            const float4* S4 = reinterpret_cast<const float4*>(buf);
            float4* G4 = state_out ? reinterpret_cast<float4*>(state_out + h * stride) : nullptr;
            const float4* V4 = reinterpret_cast<const float4*>(vf);
            float4 y[kTMax], vr[kTMax];
#pragma unroll
            for (int ii = 0; ii < kTMax; ++ii) {
                y[ii] = make_float4(0.f, 0.f, 0.f, 0.f);
                vr[ii] = ii < T ? V4[ii * kDV4w + cg] : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            for (int r = rs; r < F; r += kWGmThreads / kDV4w) {
                float4 s = S4[r * kDV4w + cg];
                const float4* cq = reinterpret_cast<const float4*>(pq + r * Tp);
                const float4* ck = reinterpret_cast<const float4*>(pk + r * Tp);
#pragma unroll
                for (int i4 = 0; i4 < kTMax / 4; ++i4) {
                    if (4 * i4 < T) {
                        const float4 c = cq[i4];
                        const float cc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            y[4 * i4 + u].x = fmaf(cc[u], s.x, y[4 * i4 + u].x);
                            y[4 * i4 + u].y = fmaf(cc[u], s.y, y[4 * i4 + u].y);
                            y[4 * i4 + u].z = fmaf(cc[u], s.z, y[4 * i4 + u].z);
                            y[4 * i4 + u].w = fmaf(cc[u], s.w, y[4 * i4 + u].w);
                        }
                    }
                }
                if (G4) {
#pragma unroll
                    for (int j4 = 0; j4 < kTMax / 4; ++j4) {
                        if (4 * j4 < T) {  // padded tokens have coefficient 0 and v rows of zeros
                            const float4 a = ck[j4];
                            const float aa[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                            for (int u = 0; u < 4; ++u) {
                                s.x = fmaf(aa[u], vr[4 * j4 + u].x, s.x);
                                s.y = fmaf(aa[u], vr[4 * j4 + u].y, s.y);
                                s.z = fmaf(aa[u], vr[4 * j4 + u].z, s.z);
                                s.w = fmaf(aa[u], vr[4 * j4 + u].w, s.w);
                            }
                        }
                    }
                    G4[r * kDV4w + cg] = s;
                }
            }
            TA_PHASE_ACC(p_walk, p_t);
            TA_PHASE_T0(p_t);
            // the z column: token zi's read-out over row set zs, and the
            // update of each row's normaliser
            const float* Z = reinterpret_cast<const float*>(buf) + (int64_t)F * kDVw;
            float* GZ = state_out ? state_out + h * stride + (int64_t)F * kDVw : nullptr;
            float yz = 0.f;
            if (zi < T)
                for (int f = zs; f < F; f += kWGmThreads / 16) yz = fmaf(pq[f * Tp + zi], Z[f], yz);
            if (GZ) {
                for (int f = t; f < F; f += kWGmThreads) {
                    float z = Z[f];
                    const float4* c4 = reinterpret_cast<const float4*>(pk + f * Tp);
                    for (int j4 = 0; j4 < Tp4; ++j4) {
                        const float4 c = c4[j4];
                        z += (c.x + c.y) + (c.z + c.w);
                    }
                    GZ[f] = z;
                }
                // the state's padding stays zero
                for (int64_t e = (int64_t)F * (kDVw + 1) + t; e < stride; e += kWGmThreads) state_out[h * stride + e] = 0.f;
            }
            // the buffer and the coefficients have been read: hand the buffer
            // back, and reuse the coefficient space for the column partials
            ptx::fence_proxy_async_smem();
            wgm_sync(wg);
            TA_PHASE_ACC(p_z, p_t);
            TA_PHASE_T0(p_t);
            if (t == 0 && i + kWGm < nheads) issue(i + kWGm);
            float4* red4 = reinterpret_cast<float4*>(red);
#pragma unroll
            for (int ii = 0; ii < kTMax; ++ii)
                if (ii < T) red4[(rs * T + ii) * kDV4w + cg] = y[ii];
            zr[zs * kTMax + zi] = yz;
            wgm_sync(wg);
            TA_PHASE_ACC(p_red, p_t);
            TA_PHASE_T0(p_t);
            for (int e = t; e < T * kDVw; e += kWGmThreads) {
                const int ii = e / kDVw, c = e % kDVw;
                float acc = 0.f, den = 0.f;
#pragma unroll
                for (int w = 0; w < kWGmThreads / kDV4w; ++w) {
                    acc += red[(w * T + ii) * kDVw + c];
                    den += zr[w * kTMax + ii];
                }
                for (int j = 0; j <= ii; ++j) {
                    const float w = P[ii * kTMax + j];
                    acc = fmaf(w, vf[j * kDVw + c], acc);
                    den += w;
                }
                out[(h * T + ii) * kDVw + c] = acc / den;
            }
            wgm_sync(wg);  // the area is rewritten only after every thread is done with it
            TA_PHASE_ACC(p_out, p_t);
        }
        TA_PHASE_PUT(0, 1 + 6 * wg, t == 0, p_wait);
        TA_PHASE_PUT(0, 2 + 6 * wg, t == 0, p_prep);
        TA_PHASE_PUT(0, 3 + 6 * wg, t == 0, p_walk);
        TA_PHASE_PUT(0, 4 + 6 * wg, t == 0, p_z);
        TA_PHASE_PUT(0, 5 + 6 * wg, t == 0, p_red);
        TA_PHASE_PUT(0, 6 + 6 * wg, t == 0, p_out);
    }
    __syncthreads();
    TA_PHASE(0, 0, tid == 0);
    if (tid == 0 && s_bad) atomicOr(err, kErrDecodeLoad);
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

// The persistent form, when it applies (else cudaErrorNotSupported).
template <typename Tin>
cudaError_t launch_multi_ws(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* state_out,
                            float* out, int BH, int T, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                            cudaStream_t stream) {
    // features of degree <= 2 only (always the case for F <= 256 at the supported d_k)
    if (dv != kDVw || F > 256 || n > 3 || d > 32 || ((int64_t)T * d * sizeof(Tin)) % 16 != 0) return cudaErrorNotSupported;
    static std::once_flag once[kMaxDevices];
    static cudaError_t set_err[kMaxDevices];
    static int num_sms[kMaxDevices];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        set_err[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(decode_multi_ws_kernel<Tin>),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDynWSm);
        if (set_err[dev] == cudaSuccess)
            set_err[dev] = cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    if (set_err[dev] != cudaSuccess) return set_err[dev];
    if (BH < 2 * num_sms[dev]) return cudaErrorNotSupported;  // few heads: one CTA per head is as good
    const uint32_t bytes = (uint32_t)((F * (dv + 1) * 4 + 15) / 16 * 16);
    const MultiWsLayout L = multi_ws_layout(T, d, (int)F, bytes, (uint32_t)sizeof(Tin));
    const size_t dyn = L.bytes;
    if (dyn > kMaxDynWSm) return cudaErrorNotSupported;
    unsigned int* err = device_error_word();
    if (!err) return cudaErrorNotSupported;
    const int grid = num_sms[dev] < BH ? num_sms[dev] : BH;
    cudaError_t e = cudaSuccess;
    TA_TIMED(stream, "decode_multi_ws_kernel",
             e = launch_maybe_pdl(decode_multi_ws_kernel<Tin>, dim3(grid), dim3(kThreadsWSm), dyn, stream, true, q, k,
                                  v, state_in, state_out, out, BH, T, d, n, tau, (int)F, stride, bytes, err));
    return e != cudaSuccess ? e : cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_decode_multi(const Tin* q, const Tin* k, const Tin* v, const float* state_in, float* state_out,
                                float* out, int BH, int T, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                                cudaStream_t stream) {
    if (T < 1 || T > kTMax || F > 1024) return cudaErrorNotSupported;
    // Above 8 tokens per call the tensor-core kernel is the faster one on
    // the decode workload (its cost is nearly flat in T; the CUDA-core row
    // walk grows with T): 35.6 / 35.7 us at T = 8, 53.6 / 37.1 us at T = 16.
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
        if (T > kTcMinTokens) {
            const cudaError_t et = launch_decode_multi_tc(q, k, v, state_in, state_out, out, BH, T, d, dv, n, tau,
                                                          F, stride, stream);
            if (et != cudaErrorNotSupported) return et;
        }
    }
    {
        const cudaError_t ew = launch_multi_ws(q, k, v, state_in, state_out, out, BH, T, d, dv, n, tau, F, stride,
                                               stream);
        if (ew != cudaErrorNotSupported) return ew;
    }
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
