// Chunked causal prefill on CUDA cores, fp32 arithmetic throughout.  This is
// the fp32 path of the library and the path for shapes without a tensor-core
// specialisation.
//
// Method (arXiv 2610.20637, abstract): states are additive across chunks, so
// prefill is a scan.  Tokens are cut into groups of G; then
//   A. group_state: dS_g = sum_{t in g} phi(k_t) [v_t | 1]^T    (per group)
//   B. scan:        S_<g = sum_{g' < g} dS_g', in place; the total is the
//                   final state                                   (per head)
//   C. chunk_out:   for 64 query tokens of group g,
//                   y = sum_{j in g, j <= i} K(tau q_i.k_j) [v_j | 1]
//                     + (c (.) phi(q_i))^T S_<g,   o = y[:d_v] / y[d_v].
// Inside a group the kernel is evaluated pairwise; across groups through the
// state.  G is picked so the pairwise part costs about half the read-out.
#include <algorithm>

#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace ta {

namespace {

constexpr int kC = 64;         // tokens per sub-chunk
constexpr int kThreads = 256;
constexpr int kFTA = 64;       // features per group_state CTA
constexpr int kFTC = 32;       // features per read-out tile in chunk_out

// ---------------------------------------------------------------- A
template <typename Tin, int RPT>
__global__ void __launch_bounds__(kThreads)
group_state_kernel(const Tin* __restrict__ k, const Tin* __restrict__ v, float* __restrict__ W,
                   int N, int d, int dv, int n, int G, int NG, int F, int64_t stride) {
    extern __shared__ float4 sm4[];
    float* ks = reinterpret_cast<float*>(sm4);   // [kC][d]
    float* vs = ks + kC * ((d + 3) & ~3);         // [kC][dv]
    float* ph = vs + kC * dv;                     // [kC][kFTA]
    FeatDesc* ds = reinterpret_cast<FeatDesc*>(ph + kC * kFTA);

    const int g = blockIdx.x, bh = blockIdx.z;
    const int f0 = blockIdx.y * kFTA;
    const int nf = min(kFTA, F - f0);
    const int tid = threadIdx.x;
    const int dv4 = dv >> 2;
    const int rsets = kThreads / dv4;
    const int cg = tid % dv4, rs = tid / dv4;
    const bool active = rs < rsets;
    const int dpad = (d + 3) & ~3;

    if (tid < nf) ds[tid] = get_desc(feat_table(d, n), d, n, f0 + tid, 0.f, nullptr, false);

    float4 acc[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    float zacc = 0.f;

    const int64_t tb = (int64_t)g * G;
    const int64_t te = min64(N, tb + G);
    const Tin* kb = k + (int64_t)bh * N * d;
    const Tin* vb = v + (int64_t)bh * N * dv;
    for (int64_t c0 = tb; c0 < te; c0 += kC) {
        const int nt = (int)min64(kC, te - c0);
        __syncthreads();
        for (int i = tid; i < nt * d; i += kThreads) ks[(i / d) * dpad + i % d] = ldf(kb + c0 * d + i);
        for (int i = tid; i < nt * dv; i += kThreads) vs[i] = ldf(vb + c0 * dv + i);
        __syncthreads();
        for (int i = tid; i < nt * kFTA; i += kThreads) {
            const int t = i / kFTA, f = i % kFTA;
            ph[i] = f < nf ? eval_desc(ds[f], ks + t * dpad) : 0.f;
        }
        __syncthreads();
        if (active) {
            for (int t = 0; t < nt; ++t) {
                const float4 v4 = *reinterpret_cast<const float4*>(vs + t * dv + cg * 4);
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const int r = rs + i * rsets;
                    if (r < nf) {
                        const float a = ph[t * kFTA + r];
                        acc[i].x = fmaf(a, v4.x, acc[i].x);
                        acc[i].y = fmaf(a, v4.y, acc[i].y);
                        acc[i].z = fmaf(a, v4.z, acc[i].z);
                        acc[i].w = fmaf(a, v4.w, acc[i].w);
                    }
                }
            }
        }
        if (tid < nf)
            for (int t = 0; t < nt; ++t) zacc += ph[t * kFTA + tid];
    }
    float* Wg = W + ((int64_t)bh * NG + g) * stride;
    if (active) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) {
            const int r = rs + i * rsets;
            if (r < nf) *reinterpret_cast<float4*>(Wg + (int64_t)(f0 + r) * dv + cg * 4) = acc[i];
        }
    }
    if (tid < nf) Wg[(int64_t)F * dv + f0 + tid] = zacc;
}

// ---------------------------------------------------------------- B
// Exclusive scan over the NG group states of a head, in place, starting from
// a carried-in state (or zero).  A block covers kScanCols float4 columns of
// one head; its kScanParts warp groups take consecutive quarters of the
// groups, keep all their loads in flight, and combine the quarters' totals
// through shared memory.  The total is the state after every group; elements
// past F*(d_v+1) (padding, never written by the producers) come out as zeros.
constexpr int kScanCols = 32;                        // float4 columns per block
constexpr int kScanParts = 4;                        // group quarters per block
constexpr int kScanThreads = kScanCols * kScanParts; // 128
constexpr int kScanRun = 8;                          // loads in flight per thread

__global__ void __launch_bounds__(kScanThreads, 8)
scan_kernel(float* __restrict__ W, const float* __restrict__ state_in, float* __restrict__ state_out, int NG,
            int64_t stride, int64_t used) {
    // the group states come from the previous kernel; the next one may start
    // its independent work as soon as this grid is resident
    ptx::pdl_wait_primary();
    ptx::pdl_launch_dependents();
    __shared__ float4 part_sum[kScanParts][kScanCols];
    const int bh = blockIdx.y;
    const int col = threadIdx.x % kScanCols, part = threadIdx.x / kScanCols;
    const int64_t e4 = (int64_t)blockIdx.x * kScanCols + col;
    const int64_t s4 = stride / 4;
    const bool live = e4 < s4;
    const int per = (NG + kScanParts - 1) / kScanParts;
    const int g_begin = min(NG, part * per), g_end = min(NG, g_begin + per);
    float4* base = reinterpret_cast<float4*>(W + (int64_t)bh * NG * stride) + e4;
    const int64_t e = e4 * 4;
    auto mask_tail = [&](float4 r) {
        if (e + 0 >= used) r.x = 0.f;
        if (e + 1 >= used) r.y = 0.f;
        if (e + 2 >= used) r.z = 0.f;
        if (e + 3 >= used) r.w = 0.f;
        return r;
    };

    // pass 1: this quarter's total
    float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int g0 = g_begin; g0 < g_end; g0 += kScanRun) {
        float4 x[kScanRun];
#pragma unroll
        for (int j = 0; j < kScanRun; ++j)
            if (live && g0 + j < g_end) x[j] = base[(int64_t)(g0 + j) * s4];
#pragma unroll
        for (int j = 0; j < kScanRun; ++j)
            if (live && g0 + j < g_end) {
                tot.x += x[j].x;
                tot.y += x[j].y;
                tot.z += x[j].z;
                tot.w += x[j].w;
            }
    }
    part_sum[part][col] = tot;
    __syncthreads();
    // the carried state plus the earlier quarters
    float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
    if (state_in && live) run = mask_tail(reinterpret_cast<const float4*>(state_in + (int64_t)bh * stride)[e4]);
    for (int p = 0; p < part; ++p) {
        const float4 t = part_sum[p][col];
        run.x += t.x;
        run.y += t.y;
        run.z += t.z;
        run.w += t.w;
    }
    // pass 2: exclusive prefixes (these loads hit L2: pass 1 just read them)
    for (int g0 = g_begin; g0 < g_end; g0 += kScanRun) {
        float4 x[kScanRun];
#pragma unroll
        for (int j = 0; j < kScanRun; ++j)
            if (live && g0 + j < g_end) x[j] = base[(int64_t)(g0 + j) * s4];
#pragma unroll
        for (int j = 0; j < kScanRun; ++j) {
            if (live && g0 + j < g_end) {
                base[(int64_t)(g0 + j) * s4] = run;
                run.x += x[j].x;
                run.y += x[j].y;
                run.z += x[j].z;
                run.w += x[j].w;
            }
        }
    }
    // after its own quarter the last part holds the total
    if (state_out && live && part == kScanParts - 1)
        reinterpret_cast<float4*>(state_out + (int64_t)bh * stride)[e4] = mask_tail(run);
}

// ---------------------------------------------------------------- C
struct OutSmem {
    int dq;  // row stride of qs/ks (d + 1)
    size_t qs, ks, vs, P, phq, Ss, zs, ds, total;
};

__host__ __device__ inline OutSmem out_smem_layout(int d) {
    OutSmem L;
    L.dq = d + 1;
    size_t o = 0;
    L.qs = o; o += (size_t)kC * L.dq;
    L.ks = o; o += (size_t)kC * L.dq;
    o = (o + 3) & ~(size_t)3;
    L.vs = o; o += (size_t)kC * 64;
    L.P = o; o += (size_t)kC * (kC + 1);
    L.phq = o; o += (size_t)kC * (kFTC + 1);
    o = (o + 3) & ~(size_t)3;
    L.Ss = o; o += (size_t)kFTC * 64;
    L.zs = o; o += kFTC;
    L.ds = o; o += (size_t)kFTC * (sizeof(FeatDesc) / sizeof(float));
    L.total = o * sizeof(float);
    return L;
}

template <typename Tin>
__global__ void __launch_bounds__(kThreads)
chunk_out_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                 const float* __restrict__ W, float* __restrict__ out, int N, int d, int dv, int n,
                 float tau, int G, int NG, int F, int64_t stride, int carried) {
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    const OutSmem L = out_smem_layout(d);
    float* qs = sm + L.qs;
    float* ks = sm + L.ks;
    float* vs = sm + L.vs;
    float* P = sm + L.P;
    float* phq = sm + L.phq;
    float* Ss = sm + L.Ss;
    float* zs = sm + L.zs;
    FeatDesc* ds = reinterpret_cast<FeatDesc*>(sm + L.ds);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int i = tid >> 2, qq = tid & 3;
    const int bh = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kC;
    const int nq = (int)min64(kC, N - q0);
    const int g = (int)(q0 / G);
    const int64_t gs = (int64_t)g * G;
    const int dq = L.dq;

    const Tin* qb = q + (int64_t)bh * N * d;
    const Tin* kb = k + (int64_t)bh * N * d;
    const Tin* vb = v + (int64_t)bh * N * dv;
    const PackedFeat* tab = feat_table(d, n);
    __shared__ float qc[kMaxN];
    if (tid < n) qc[tid] = query_coeff(tid, tau);
    for (int e = tid; e < kC * d; e += kThreads) {
        const int r = e / d, s = e % d;
        qs[r * dq + s] = r < nq ? ldf(qb + (q0 + r) * d + s) : 0.f;
    }

    for (int cb = 0; cb < dv; cb += 64) {
        const int cw = min(64, dv - cb);
        float acc[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) acc[c] = 0.f;
        float den = 0.f;

        // pairwise part over the keys of this group up to the diagonal
        for (int64_t k0 = gs; k0 <= q0; k0 += kC) {
            const int nk = (int)min64(kC, N - k0);
            __syncthreads();
            for (int e = tid; e < nk * d; e += kThreads) {
                const int r = e / d, s = e % d;
                ks[r * dq + s] = ldf(kb + (k0 + r) * d + s);
            }
            for (int e = tid; e < nk * cw; e += kThreads) {
                const int r = e / cw, c = e % cw;
                vs[r * 64 + c] = ldf(vb + (k0 + r) * dv + cb + c);
            }
            __syncthreads();
#pragma unroll 4
            for (int jj = 0; jj < 16; ++jj) {
                const int j = qq * 16 + jj;
                float p = 0.f;
                if (i < nq && j < nk && k0 + j <= q0 + i) {
                    float dot = 0.f;
                    for (int s = 0; s < d; ++s) dot = fmaf(qs[i * dq + s], ks[j * dq + s], dot);
                    p = taylor_kernel(tau * dot, n);
                }
                P[i * (kC + 1) + j] = p;
            }
            __syncthreads();
            for (int j = 0; j < nk; ++j) {
                const float p = P[i * (kC + 1) + j];
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] = fmaf(p, vs[j * 64 + qq * 16 + c], acc[c]);
                if (qq == 0) den += p;
            }
        }

        // across groups, through the exclusive prefix state S_<g (which holds
        // the carried-in state when the sequence continues one)
        if (g > 0 || carried) {
            const float* Sg = W + ((int64_t)bh * NG + g) * stride;
            for (int f0 = 0; f0 < F; f0 += kFTC) {
                const int nf = min(kFTC, F - f0);
                __syncthreads();
                if (tid < nf) ds[tid] = get_desc(tab, d, n, f0 + tid, tau, qc, true);
                for (int e = tid; e < nf * cw; e += kThreads) {
                    const int r = e / cw, c = e % cw;
                    Ss[r * 64 + c] = Sg[(int64_t)(f0 + r) * dv + cb + c];
                }
                if (tid < nf) zs[tid] = Sg[(int64_t)F * dv + f0 + tid];
                __syncthreads();
                for (int e = tid; e < kC * kFTC; e += kThreads) {
                    const int r = e / kFTC, f = e % kFTC;
                    phq[r * (kFTC + 1) + f] = (r < nq && f < nf) ? eval_desc(ds[f], qs + r * dq) : 0.f;
                }
                __syncthreads();
                for (int f = 0; f < nf; ++f) {
                    const float p = phq[i * (kFTC + 1) + f];
#pragma unroll
                    for (int c = 0; c < 16; ++c) acc[c] = fmaf(p, Ss[f * 64 + qq * 16 + c], acc[c]);
                    if (qq == 0) den = fmaf(p, zs[f], den);
                }
            }
        }

        den = __shfl_sync(0xffffffffu, den, lane & ~3);
        if (i < nq) {
            float* o = out + ((int64_t)bh * N + q0 + i) * dv + cb + qq * 16;
#pragma unroll
            for (int c = 0; c < 16; ++c)
                if (qq * 16 + c < cw) o[c] = acc[c] / den;
        }
    }
}

// ---------------------------------------------------------------- C'
// Output kernel of the mean-centred softmax expansion (Su Jianlin, "Taylor
// expansions of logsumexp and softmax", kexue.fm translation 11814, sections
// "Calculating the Gradient" and "Linear Attention"), over the same group
// states as C (those of the n = 3 Taylor kernel: their degree-0, 1 and 2 rows
// hold every prefix sum the expansion needs).  For query i the three
// per-degree read-outs R_m = sum_{j <= i} (q_i.k_j)^m [v_j | 1] (no tau, no
// 1/m!) are accumulated apart: pairwise inside the group, through
// phi_m(q_i)^T S_<g,m across groups.  Then, per column,
//   n = R_0[z], V = R_0[v], qkbar = R_1[z] / n,
//   sum a v   = tau (R_1[v] - qkbar V),
//   sum a^2 v = tau^2 (R_2[v] - 2 qkbar R_1[v] + qkbar^2 V),
//   sum a^2   = tau^2 (R_2[z] - n qkbar^2),
//   o = V/n + (sum a v)/n  [+ (sum a^2 v - (sum a^2) V/n) / (2n) at order 2].
template <typename Tin>
__global__ void __launch_bounds__(kThreads)
centred_chunk_out_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
                         const float* __restrict__ W, float* __restrict__ out, int N, int d, int dv, int order,
                         float tau, int G, int NG, int F, int64_t stride, int carried) {
    extern __shared__ float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    const OutSmem L = out_smem_layout(d);
    float* qs = sm + L.qs;
    float* ks = sm + L.ks;
    float* vs = sm + L.vs;
    float* P = sm + L.P;
    float* phq = sm + L.phq;
    float* Ss = sm + L.Ss;
    float* zs = sm + L.zs;
    FeatDesc* ds = reinterpret_cast<FeatDesc*>(sm + L.ds);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int i = tid >> 2, qq = tid & 3;
    const int bh = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kC;
    const int nq = (int)min64(kC, N - q0);
    const int g = (int)(q0 / G);
    const int64_t gs = (int64_t)g * G;
    const int dq = L.dq;

    const Tin* qb = q + (int64_t)bh * N * d;
    const Tin* kb = k + (int64_t)bh * N * d;
    const Tin* vb = v + (int64_t)bh * N * dv;
    const PackedFeat* tab = feat_table(d, 3);
    for (int e = tid; e < kC * d; e += kThreads) {
        const int r = e / d, s = e % d;
        qs[r * dq + s] = r < nq ? ldf(qb + (q0 + r) * d + s) : 0.f;
    }

    for (int cb = 0; cb < dv; cb += 64) {
        const int cw = min(64, dv - cb);
        float a0[16], a1[16], a2[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) a0[c] = a1[c] = a2[c] = 0.f;
        float z0 = 0.f, z1 = 0.f, z2 = 0.f;

        // pairwise part over the keys of this group up to the diagonal: the
        // raw score s = q.k_j, its square, and 1
        for (int64_t k0 = gs; k0 <= q0; k0 += kC) {
            const int nk = (int)min64(kC, N - k0);
            __syncthreads();
            for (int e = tid; e < nk * d; e += kThreads) {
                const int r = e / d, s = e % d;
                ks[r * dq + s] = ldf(kb + (k0 + r) * d + s);
            }
            for (int e = tid; e < nk * cw; e += kThreads) {
                const int r = e / cw, c = e % cw;
                vs[r * 64 + c] = ldf(vb + (k0 + r) * dv + cb + c);
            }
            __syncthreads();
#pragma unroll 4
            for (int jj = 0; jj < 16; ++jj) {
                const int j = qq * 16 + jj;
                float dot = 0.f;
                if (i < nq && j < nk)
                    for (int s = 0; s < d; ++s) dot = fmaf(qs[i * dq + s], ks[j * dq + s], dot);
                P[i * (kC + 1) + j] = dot;
            }
            __syncthreads();
            // keys j <= i of this tile (all of them below the diagonal tile)
            const int jn = i < nq ? (int)min64(nk, q0 + i - k0 + 1) : 0;
            for (int j = 0; j < jn; ++j) {
                const float s1 = P[i * (kC + 1) + j];
                const float s2 = s1 * s1;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const float x = vs[j * 64 + qq * 16 + c];
                    a0[c] += x;
                    a1[c] = fmaf(s1, x, a1[c]);
                    a2[c] = fmaf(s2, x, a2[c]);
                }
                if (qq == 0) {
                    z0 += 1.f;
                    z1 += s1;
                    z2 += s2;
                }
            }
        }

        // across groups, through the exclusive prefix state S_<g: each
        // feature's read-out goes to the accumulator of its degree
        if (g > 0 || carried) {
            const float* Sg = W + ((int64_t)bh * NG + g) * stride;
            for (int f0 = 0; f0 < F; f0 += kFTC) {
                const int nf = min(kFTC, F - f0);
                __syncthreads();
                if (tid < nf) ds[tid] = get_desc(tab, d, 3, f0 + tid, 1.f, nullptr, false);
                for (int e = tid; e < nf * cw; e += kThreads) {
                    const int r = e / cw, c = e % cw;
                    Ss[r * 64 + c] = Sg[(int64_t)(f0 + r) * dv + cb + c];
                }
                if (tid < nf) zs[tid] = Sg[(int64_t)F * dv + f0 + tid];
                __syncthreads();
                for (int e = tid; e < kC * kFTC; e += kThreads) {
                    const int r = e / kFTC, f = e % kFTC;
                    phq[r * (kFTC + 1) + f] = (r < nq && f < nf) ? eval_desc(ds[f], qs + r * dq) : 0.f;
                }
                __syncthreads();
                for (int f = 0; f < nf; ++f) {
                    const float p = phq[i * (kFTC + 1) + f];
                    const int m = ds[f].m;  // the same for every thread
                    const float* sr = Ss + f * 64 + qq * 16;
                    if (m == 0) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) a0[c] = fmaf(p, sr[c], a0[c]);
                    } else if (m == 1) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) a1[c] = fmaf(p, sr[c], a1[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 16; ++c) a2[c] = fmaf(p, sr[c], a2[c]);
                    }
                    if (qq == 0) {
                        const float pz = p * zs[f];
                        if (m == 0) z0 += pz;
                        else if (m == 1) z1 += pz;
                        else z2 += pz;
                    }
                }
            }
        }

        z0 = __shfl_sync(0xffffffffu, z0, lane & ~3);
        z1 = __shfl_sync(0xffffffffu, z1, lane & ~3);
        z2 = __shfl_sync(0xffffffffu, z2, lane & ~3);
        if (i < nq) {
            const float n = z0, qkbar = z1 / n, t2 = tau * tau;
            const float sum_a2 = t2 * (z2 - n * qkbar * qkbar);
            float* o = out + ((int64_t)bh * N + q0 + i) * dv + cb + qq * 16;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                if (qq * 16 + c < cw) {
                    const float V = a0[c];
                    float r = V / n + tau * (a1[c] - qkbar * V) / n;
                    if (order >= 2) {
                        const float sum_a2v = t2 * (a2[c] - 2.0f * qkbar * a1[c] + qkbar * qkbar * V);
                        r += (sum_a2v - sum_a2 * V / n) / (2.0f * n);
                    }
                    o[c] = r;
                }
            }
        }
    }
}

template <typename T>
cudaError_t set_smem(T* fn, size_t bytes) {
    return cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

int pow2ceil(int64_t x) {
    int p = 1;
    while (p < x && p < (1 << 30)) p <<= 1;
    return p;
}

}  // namespace

CcPlan plan_prefill_cc(int BH, int N, int d, int dv, int n, int64_t F, int64_t stride) {
    (void)n;
    CcPlan p;
    // pairwise cost per token ~ G (d + dv + 1); read-out ~ 2 F (dv + 1)
    int64_t want = (F * (dv + 1)) / (d + dv + 1);
    int G = pow2ceil(std::max<int64_t>(want, 1));
    G = std::max(G, kC);
    G = std::min(G, 4096);
    G = std::min(G, std::max(kC, pow2ceil(N)));
    p.G = G;
    p.NG = N > 0 ? (N + G - 1) / G : 0;
    p.ws_bytes = (size_t)BH * (size_t)p.NG * (size_t)stride * sizeof(float);
    return p;
}

// A and B: per-group states of (d, n) and their exclusive scan, in W.
template <typename Tin>
cudaError_t launch_group_states(const Tin* k, const Tin* v, const float* state_in, float* state_out, float* W,
                                const CcPlan& plan, int BH, int N, int d, int dv, int n, int64_t F, int64_t stride,
                                cudaStream_t stream) {
    cudaError_t e;
    // A
    const int dv4 = dv / 4;
    const int rsets = kThreads / dv4;
    const int need = (kFTA + rsets - 1) / rsets;
    const size_t smA = (size_t)(kC * ((d + 3) & ~3) + kC * dv + kC * kFTA) * sizeof(float) +
                       kFTA * sizeof(FeatDesc);
    const dim3 gA(plan.NG, (unsigned)((F + kFTA - 1) / kFTA), BH);
#define TA_LAUNCH_A(R)                                                                     \
    do {                                                                                   \
        auto fn = group_state_kernel<Tin, R>;                                              \
        if ((e = set_smem(fn, smA)) != cudaSuccess) return e;                              \
        TA_TIMED(stream, "cc_group_state_kernel",                                          \
                 fn<<<gA, kThreads, smA, stream>>>(k, v, W, N, d, dv, n, plan.G, plan.NG,  \
                                                   (int)F, stride));                       \
    } while (0)
    if (need <= 1) TA_LAUNCH_A(1);
    else if (need <= 2) TA_LAUNCH_A(2);
    else if (need <= 4) TA_LAUNCH_A(4);
    else if (need <= 8) TA_LAUNCH_A(8);
    else TA_LAUNCH_A(16);
#undef TA_LAUNCH_A
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // B
    const dim3 gB((unsigned)((stride / 4 + kScanCols - 1) / kScanCols), BH);
    TA_TIMED(stream, "cc_scan_kernel",
             scan_kernel<<<gB, kScanThreads, 0, stream>>>(W, state_in, state_out, plan.NG, stride, F * (dv + 1)));
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_prefill_cc(const Tin* q, const Tin* k, const Tin* v, float* out,
                              const float* state_in, float* state_out, float* W, const CcPlan& plan,
                              int BH, int N, int d, int dv, int n, float tau, int64_t F, int64_t stride,
                              cudaStream_t stream) {
    if (BH == 0 || N == 0) return cudaSuccess;
    cudaError_t e;
    // a single group with no state in or out needs neither A nor B
    const bool need_states = plan.NG > 1 || state_out != nullptr || state_in != nullptr;
    if (need_states) {
        e = launch_group_states(k, v, state_in, state_out, W, plan, BH, N, d, dv, n, F, stride, stream);
        if (e != cudaSuccess) return e;
    }
    // C
    const OutSmem L = out_smem_layout(d);
    auto fc = chunk_out_kernel<Tin>;
    if ((e = set_smem(fc, L.total)) != cudaSuccess) return e;
    const dim3 gC((unsigned)((N + kC - 1) / kC), BH);
    TA_TIMED(stream, "cc_chunk_out_kernel",
             fc<<<gC, kThreads, L.total, stream>>>(q, k, v, W, out, N, d, dv, n, tau, plan.G, plan.NG,
                                                   (int)F, stride, state_in != nullptr ? 1 : 0));
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_centred_prefill_cc(const Tin* q, const Tin* k, const Tin* v, float* out,
                                      const float* state_in, float* state_out, float* W, const CcPlan& plan,
                                      int BH, int N, int d, int dv, int order, float tau, int64_t F,
                                      int64_t stride, cudaStream_t stream) {
    if (BH == 0 || N == 0) return cudaSuccess;
    cudaError_t e;
    const bool need_states = plan.NG > 1 || state_out != nullptr || state_in != nullptr;
    if (need_states) {
        e = launch_group_states(k, v, state_in, state_out, W, plan, BH, N, d, dv, 3, F, stride, stream);
        if (e != cudaSuccess) return e;
    }
    const OutSmem L = out_smem_layout(d);
    auto fc = centred_chunk_out_kernel<Tin>;
    if ((e = set_smem(fc, L.total)) != cudaSuccess) return e;
    const dim3 gC((unsigned)((N + kC - 1) / kC), BH);
    TA_TIMED(stream, "cc_centred_chunk_out_kernel",
             fc<<<gC, kThreads, L.total, stream>>>(q, k, v, W, out, N, d, dv, order, tau, plan.G, plan.NG,
                                                   (int)F, stride, state_in != nullptr ? 1 : 0));
    return cudaGetLastError();
}

cudaError_t launch_state_scan(float* W, const float* state_in, float* state_out, int BH, int NG, int64_t stride,
                              int64_t used, cudaStream_t stream, bool pdl) {
    const dim3 g((unsigned)((stride / 4 + kScanCols - 1) / kScanCols), BH);
    cudaError_t e = cudaSuccess;
    TA_TIMED(stream, "scan_kernel",
             e = launch_maybe_pdl(scan_kernel, g, dim3(kScanThreads), 0, stream, pdl, W, state_in, state_out, NG,
                                  stride, used));
    return e != cudaSuccess ? e : cudaGetLastError();
}

template cudaError_t launch_prefill_cc<float>(const float*, const float*, const float*, float*, const float*,
                                              float*, float*, const CcPlan&, int, int, int, int, int, float,
                                              int64_t, int64_t, cudaStream_t);
template cudaError_t launch_prefill_cc<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                      const __nv_bfloat16*, float*, const float*, float*,
                                                      float*, const CcPlan&, int, int, int, int, int, float,
                                                      int64_t, int64_t, cudaStream_t);
template cudaError_t launch_centred_prefill_cc<float>(const float*, const float*, const float*, float*,
                                                      const float*, float*, float*, const CcPlan&, int, int, int,
                                                      int, int, float, int64_t, int64_t, cudaStream_t);
template cudaError_t launch_centred_prefill_cc<__nv_bfloat16>(const __nv_bfloat16*, const __nv_bfloat16*,
                                                              const __nv_bfloat16*, float*, const float*, float*,
                                                              float*, const CcPlan&, int, int, int, int, int,
                                                              float, int64_t, int64_t, cudaStream_t);

}  // namespace ta
