// Chunked causal prefill on the sm_100a tensor cores for any number of
// features: d_k in {16, 32, 64}, d_v = 64, bf16 inputs.  The state does not
// fit one SM at these widths (2,145 features at d_k 64, n 3; 4,845 at d_k 16,
// n 5), so features are cut into tiles.
//
// Method (arXiv 2610.20637, abstract): the state S = sum_j phi(k_j)[v_j|1]^T
// is additive across chunks, so prefill is a scan over group states.
// Tokens are cut into groups of G (a multiple of 128); then
//   1. tcf_state_kernel (group, 128-feature tile, head):
//        dS_g[tile, :] = Phi_K[:, tile]^T (128 x G) . [V|1|0] (G x 80),
//        accumulated in TMEM over 64-token stages;
//   2. the exclusive scan over groups (shared with the other paths);
//   3. tcf_out_kernel (128 queries, head):
//        O = sum over 64-key tiles of the group up to the diagonal of
//              (poly(tau Q K^T) (.) mask) [V|1|0]
//          + sum over 64-feature tiles of (c (.) Phi_Q[:, tile]) S_<g[tile, :],
//        o = O[:, :64] / O[:, 64].
// Operands produced in fp32 (Phi_K, Phi_Q, P and S_<g) are split into hi/lo
// bf16 pairs (about 16 significant bits reach the fp32 accumulators); q, k and
// v are bf16 already.  Both kernels are software pipelined: 16-byte cp.async
// copies fill a ring of stages, the CUDA cores evaluate features (or P) for
// one stage while the tensor cores run the MMAs of the previous one, and each
// stage is handed back through an mbarrier that tcgen05.commit arrives on.
// Every wait is bounded; a timeout sets a device error bit.
#pragma once

#include <mutex>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "feat_eval.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "prefill_tc.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace ta {
namespace tc {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kTok = 64;      // tokens per state stage, keys per pairwise tile
constexpr int kFT = 128;      // features per state tile (M of the state MMA)
constexpr int kRT = 64;       // features per read-out tile (K of the read-out MMA)
constexpr int kQ = 128;       // queries per output CTA (M)
constexpr int kDV = 64;
constexpr int kNV = 80;       // [V | 1 | 0 ...]
constexpr int kThreads = 256;
constexpr uint32_t kWaitPolls = 1u << 24;

constexpr uint32_t kLboNV = (kNV / 8) * 128;    // K-group stride of an MN-major operand 80 wide
constexpr uint32_t kLboFT = (kFT / 8) * 128;    // K-group stride of an MN-major operand 128 wide
constexpr uint32_t kSbo64 = (64 / 8) * 128;     // row-group stride of a K-major operand 64 deep

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    return ptx::mbar_wait(bar, parity, kWaitPolls);
}

// Orders this thread's shared-memory writes before the tensor cores read them
// and synchronises the block; true if any thread reports a failure.
__device__ __forceinline__ bool publish(bool bad) {
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    const bool any = __syncthreads_or(bad) != 0;
    fence_after_sync();
    return any;
}

// Eight fp32 values -> hi/lo bf16 chunks stored at two operand addresses.
__device__ __forceinline__ void store_split8(const float* x, uint8_t* hi_dst, uint8_t* lo_dst) {
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(hi_dst) = hi;
    *reinterpret_cast<uint4*>(lo_dst) = lo;
}

// `rows` token rows of a [*, D] bf16 tensor into a K-major operand (rows past
// `valid` >= 1 zero-filled) by 16-byte cp.async.
template <int D>
__device__ __forceinline__ void load_rows_kmajor(uint8_t* dst, const bf16* src, int valid, int rows) {
    constexpr int KC = D / 8;
    constexpr uint32_t sbo = KC * 128;
    for (int e = threadIdx.x; e < rows * KC; e += kThreads) {
        const int r = e / KC, c = e % KC;
        const int rr = r < valid ? r : valid - 1;
        ptx::cp_async16(dst + kmaj(r, c, sbo), src + (int64_t)rr * D + c * 8, r < valid ? 16u : 0u);
    }
}

// [v | 1 | 0] rows of 64 tokens as an MN-major [K = token][N = 80] operand:
// v by cp.async, the ones column by a plain store (column group 9 stays 0).
__device__ __forceinline__ void load_v1(uint8_t* dst, const bf16* v, int valid) {
    for (int e = threadIdx.x; e < kTok * 8; e += kThreads) {
        const int r = e >> 3, c = e & 7;
        const int rr = r < valid ? r : valid - 1;
        ptx::cp_async16(dst + mnmaj(r, c, kLboNV), v + (int64_t)rr * kDV + c * 8, r < valid ? 16u : 0u);
    }
    if (threadIdx.x < kTok)
        *reinterpret_cast<uint4*>(dst + mnmaj(threadIdx.x, 8, kLboNV)) =
            make_uint4((int)threadIdx.x < valid ? 0x3F80u : 0u, 0, 0, 0);
}

__device__ __forceinline__ void zero_v1_tail(uint8_t* dst) {
    if (threadIdx.x < kTok) *reinterpret_cast<uint4*>(dst + mnmaj(threadIdx.x, 9, kLboNV)) = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------- 1. group states
// Stage: Phi_K hi/lo as MN-major [K = 64 tokens][M = 128 features], the
// [V|1|0] operand, and the k rows (K-major) the features are read from.
template <int D>
struct StateSmem {
    static constexpr uint32_t kPhi = kTok * kFT * 2;
    static constexpr uint32_t kV1 = kTok * kNV * 2;
    static constexpr uint32_t kK = kTok * D * 2;
    static constexpr uint32_t kStage = 2 * kPhi + kV1 + kK;
    static constexpr int kStages = 3;
    static constexpr uint32_t kBytes = kStages * kStage;
    static constexpr int kOutStride = kDV + 4;  // epilogue staging rows: 16-byte aligned, float4 conflict-free
    static_assert(kFT * kOutStride * 4 <= kStage, "epilogue staging fits one stage");
};

template <int D, int N>
__global__ void __launch_bounds__(kThreads, 1)
tcf_state_kernel(const bf16* __restrict__ k, const bf16* __restrict__ v, float* __restrict__ W, int Ntok, int n,
                 int F, int64_t stride, int G, int NG, unsigned int* __restrict__ err) {
    using L = StateSmem<D>;
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t bar[L::kStages];
    __shared__ uint32_t tslot;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, ft = blockIdx.y, bh = blockIdx.z;
    const int f0 = ft * kFT;
    const int nf = min(kFT, F - f0);
    const int64_t gt0 = (int64_t)g * G;
    const int gn = (int)min64(G, (int64_t)Ntok - gt0);
    const int nsub = (gn + kTok - 1) / kTok;
    const bf16* kg = k + ((int64_t)bh * Ntok + gt0) * D;
    const bf16* vg = v + ((int64_t)bh * Ntok + gt0) * kDV;

    if (tid == 0) {
        for (int i = 0; i < L::kStages; ++i) ptx::mbar_init(&bar[i], 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    for (int s = 0; s < L::kStages; ++s) zero_v1_tail(sm + s * L::kStage + 2 * L::kPhi);
    auto load_stage = [&](int s) {
        uint8_t* st = sm + (s % L::kStages) * L::kStage;
        const int valid = min(kTok, gn - s * kTok);
        load_rows_kmajor<D>(st + 2 * L::kPhi + L::kV1, kg + (int64_t)s * kTok * D, valid, kTok);
        load_v1(st + 2 * L::kPhi, vg + (int64_t)s * kTok * kDV, valid);
        ptx::cp_async_commit();
    };
    load_stage(0);
    if (nsub > 1) load_stage(1);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tacc = tslot;

    // thread -> token t of the stage, features [32 qf, 32 qf + 32) of the tile
    const int t = tid & (kTok - 1), qf = tid >> 6;
    bool bad = false;
    int issued = 0;  // stages whose MMAs were committed
    for (int s = 0; s < nsub; ++s) {
        uint8_t* st = sm + (s % L::kStages) * L::kStage;
        if (s + 1 < nsub) ptx::cp_async_wait<1>();
        else ptx::cp_async_wait<0>();
        __syncthreads();
        {
            float o[32];
            const uint8_t* rowbase = st + 2 * L::kPhi + L::kV1 + kmaj(t, 0, (D / 8) * 128);
            fe::Eval<D, N, false>::block(ft * 4 + qf, rowbase, nullptr, n, F, 0.f, o);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                store_split8(o + 8 * i, st + mnmaj(t, qf * 4 + i, kLboFT), st + L::kPhi + mnmaj(t, qf * 4 + i, kLboFT));
        }
        if (publish(bad)) {
            bad = true;
            break;
        }
        if (tid == 0) {
            const uint32_t id = idesc_bf16(kFT, kNV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < kTok / 16; ++ks) {
                const uint64_t b = smem_desc(st + 2 * L::kPhi + ks * 2 * kLboNV, kLboNV, 128);
                mma_bf16(tacc, smem_desc(st + ks * 2 * kLboFT, kLboFT, 128), b, id, (s > 0 || ks > 0) ? 1u : 0u);
                mma_bf16(tacc, smem_desc(st + L::kPhi + ks * 2 * kLboFT, kLboFT, 128), b, id, 1u);
            }
            mma_commit(&bar[s % L::kStages]);
        }
        issued = s + 1;
        // stage (s + 2) % 3 was last read by the MMAs of stage s - 1
        if (s >= 1 && !wait_bar(&bar[(s - 1) % L::kStages], ((s - 1) / L::kStages) & 1)) bad = true;
        if (s + 2 < nsub && !bad) load_stage(s + 2);
    }
    ptx::cp_async_wait<0>();
    // MMAs complete in order: the last commit covers them all
    if (issued > 0 && !wait_bar(&bar[(issued - 1) % L::kStages], ((issued - 1) / L::kStages) & 1)) bad = true;
    bad = __syncthreads_or(bad) != 0;
    fence_after_sync();

    // TMEM lane j holds feature f0 + j: columns 0..63 its S_v row, 64 its z
    float* Wg = W + ((int64_t)bh * NG + g) * stride;
    float* sOut = reinterpret_cast<float*>(sm);
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;
    if (!bad) {
        const uint32_t ta = tacc + ((uint32_t)((warp & 3) * 32) << 16);
        float r[32];
        tmem_ld32(ta + half * 32, r);
        float zz[16];
        tmem_ld16(ta + kDV, zz);
        tmem_ld_wait();
        float4* so = reinterpret_cast<float4*>(sOut + row * L::kOutStride + half * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) so[i] = make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
        if (half == 1 && row < nf) Wg[(int64_t)F * kDV + f0 + row] = zz[0];
    } else if (tid == 0) {
        atomicOr(err, kErrPrefillPipe);
    }
    fence_before_sync();
    __syncthreads();
    if (!bad) {
        float4* dst = reinterpret_cast<float4*>(Wg + (int64_t)f0 * kDV);
        for (int e = tid; e < nf * (kDV / 4); e += kThreads) {
            const int j = e / (kDV / 4), c = e % (kDV / 4);
            dst[e] = *reinterpret_cast<const float4*>(sOut + j * L::kOutStride + c * 4);
        }
    }
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tacc, 128);
    }
}

// ---------------------------------------------------------------- 3. outputs
template <int D>
struct OutSmem {
    static constexpr uint32_t kSboD = (D / 8) * 128;  // row-group stride of K-major rows of D
    static constexpr uint32_t kQop = kQ * D * 2;      // Q, K-major [128][D]
    // pairwise: ring of 3 (K tile, [V|1|0]) + 2 x (P hi, P lo)
    static constexpr uint32_t kKt = kTok * D * 2;
    static constexpr uint32_t kV1 = kTok * kNV * 2;
    static constexpr uint32_t kKV = kKt + kV1;
    static constexpr uint32_t kP = kQ * kTok * 2;     // one of hi/lo, K-major [128][64]
    static constexpr uint32_t kPbase = 3 * kKV;
    static constexpr uint32_t kPair = kPbase + 4 * kP;
    // read-out: 2 x (Phi_Q hi, lo K-major [128][64]; S hi, lo MN-major [64][80]) + fp32 S staging
    static constexpr uint32_t kA = kQ * kRT * 2;
    static constexpr uint32_t kB = kRT * kNV * 2;
    static constexpr uint32_t kRS = 2 * kA + 2 * kB;
    static constexpr uint32_t kStg = 2 * kRS;              // staging: [64][64] S_v rows then [64] z
    static constexpr uint32_t kRead = kStg + kRT * kDV * 4 + kRT * 4;
    static constexpr uint32_t kU = kPair > kRead ? kPair : kRead;
    static constexpr uint32_t kBytes = kQop + kU;
};

template <int D, int N>
__global__ void __launch_bounds__(kThreads, 1)
tcf_out_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
               const float* __restrict__ W, float* __restrict__ out, int Ntok, int n, float tau, int F,
               int64_t stride, int G, int NG, int carried, unsigned int* __restrict__ err) {
    using L = OutSmem<D>;
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t bar_sc[2], bar_pv[2], bar_ro[2], bar_st;
    __shared__ uint32_t tslot;
    uint8_t* sQ = sm;
    uint8_t* sU = sm + L::kQop;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, bh = blockIdx.y;
    const int64_t q0 = (int64_t)qt * kQ;
    const int nq = (int)min64(kQ, (int64_t)Ntok - q0);
    const int g = (int)(q0 / G);
    const int64_t gs = (int64_t)g * G;
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int64_t kend = min64(q0 + kQ, (int64_t)Ntok);
    const int T = (int)((kend - gs + kTok - 1) / kTok);  // key tiles, >= 1

    float qc[kMaxN];
#pragma unroll
    for (int m = 0; m < kMaxN; ++m) qc[m] = query_coeff(m, tau);

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&bar_sc[i], 1);
            ptx::mbar_init(&bar_pv[i], 1);
            ptx::mbar_init(&bar_ro[i], 1);
        }
        ptx::mbar_init(&bar_st, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tslot, 256);
        tmem_relinquish();
    }
    const bf16* kb = k + (int64_t)bh * Ntok * D;
    const bf16* vb = v + (int64_t)bh * Ntok * kDV;
    auto load_tile = [&](int t) {
        uint8_t* st = sU + (t % 3) * L::kKV;
        const int64_t k0 = gs + (int64_t)t * kTok;
        const int valid = (int)min64(kTok, kend - k0);
        load_rows_kmajor<D>(st, kb + k0 * D, valid, kTok);
        load_v1(st + L::kKt, vb + k0 * kDV, valid);
        ptx::cp_async_commit();
    };
    for (int s = 0; s < 3; ++s) zero_v1_tail(sU + s * L::kKV + L::kKt);
    load_rows_kmajor<D>(sQ, q + ((int64_t)bh * Ntok + q0) * D, nq, kQ);
    load_tile(0);
    if (T > 1) {
        load_tile(1);
        ptx::cp_async_wait<1>();
    } else {
        ptx::cp_async_wait<0>();
    }
    publish(false);
    const uint32_t tS = tslot, tO = tslot + 128;

    auto issue_scores = [&](int t) {
        const uint8_t* kt = sU + (t % 3) * L::kKV;
        const uint32_t id = idesc_bf16(kQ, kTok, 0, 0);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
            mma_bf16(tS + (t & 1) * kTok, smem_desc(sQ + ks * 256, 128, L::kSboD),
                     smem_desc(kt + ks * 256, 128, L::kSboD), id, ks > 0 ? 1u : 0u);
        mma_commit(&bar_sc[t & 1]);
    };
    if (tid == 0) issue_scores(0);

    bool bad = false;
    // ------------------------------------------------ pairwise part, 64-key tiles of this group
    for (int t = 0; t < T; ++t) {
        if (!wait_bar(&bar_sc[t & 1], (t >> 1) & 1)) bad = true;
        fence_after_sync();
        {
            float s32[32];
            tmem_ld32(tS + lane_off + (t & 1) * kTok + half * 32, s32);
            tmem_ld_wait();
            const int64_t k0 = gs + (int64_t)t * kTok + half * 32;
            const int64_t qi = q0 + row;
            uint8_t* ph = sU + L::kPbase + (t & 1) * 2 * L::kP;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float x = s32[g8 * 8 + e];
                    float w;
                    if constexpr (N > 0) {
                        w = qc[N - 1];
#pragma unroll
                        for (int m = N - 2; m >= 0; --m) w = fmaf(w, x, qc[m]);
                    } else {
                        w = qc[n - 1];
                        for (int m = n - 2; m >= 0; --m) w = fmaf(w, x, qc[m]);
                    }
                    const int64_t kj = k0 + g8 * 8 + e;
                    p[e] = (kj <= qi && kj < kend && row < nq) ? w : 0.f;
                }
                const uint32_t off = kmaj(row, half * 4 + g8, kSbo64);
                store_split8(p, ph + off, ph + L::kP + off);
            }
        }
        if (t + 1 < T) ptx::cp_async_wait<0>();  // key tile t + 1 resident
        if (publish(bad)) {
            bad = true;
            break;
        }
        if (tid == 0) {
            const uint8_t* ph = sU + L::kPbase + (t & 1) * 2 * L::kP;
            const uint8_t* v1 = sU + (t % 3) * L::kKV + L::kKt;
            const uint32_t id = idesc_bf16(kQ, kNV, 0, 1);
#pragma unroll
            for (int ks = 0; ks < kTok / 16; ++ks) {
                const uint64_t b = smem_desc(v1 + ks * 2 * kLboNV, kLboNV, 128);
                mma_bf16(tO, smem_desc(ph + ks * 256, 128, kSbo64), b, id, (t > 0 || ks > 0) ? 1u : 0u);
                mma_bf16(tO, smem_desc(ph + L::kP + ks * 256, 128, kSbo64), b, id, 1u);
            }
            mma_commit(&bar_pv[t & 1]);
            if (t + 1 < T) issue_scores(t + 1);
        }
        // ring slot (t + 2) % 3 and P buffer (t + 1) & 1 were last read by PV(t - 1)
        if (t >= 1 && !wait_bar(&bar_pv[(t - 1) & 1], ((t - 1) >> 1) & 1)) bad = true;
        if (t + 2 < T && !bad) load_tile(t + 2);
    }
    ptx::cp_async_wait<0>();
    if (!bad && !wait_bar(&bar_pv[(T - 1) & 1], ((T - 1) >> 1) & 1)) bad = true;
    bad = __syncthreads_or(bad) != 0;
    fence_after_sync();

    // ------------------------------------------------ read-out through S_<g, 64-feature tiles
    ptx::pdl_wait_primary();  // the scan over group states has completed
    const int R = (F + kRT - 1) / kRT;
    int ro_issued = 0;
    if (!bad && (g > 0 || carried)) {
        const float* Sg = W + ((int64_t)bh * NG + g) * stride;
        float* stg = reinterpret_cast<float*>(sU + L::kStg);
        float* stg_z = stg + kRT * kDV;
        auto fetch_s = [&](int r) {  // S_v rows of tile r by one bulk copy, z by plain loads
            const int fr = r * kRT, nr = min(kRT, F - fr);
            if (tid == 0) {
                ptx::mbar_arrive_expect_tx(&bar_st, (uint32_t)nr * kDV * 4u);
                ptx::bulk_g2s(stg, Sg + (int64_t)fr * kDV, (uint32_t)nr * kDV * 4u, &bar_st);
            }
            if (tid < kRT) stg_z[tid] = tid < nr ? __ldg(Sg + (int64_t)F * kDV + fr + tid) : 0.f;
        };
        fetch_s(0);
        for (int r = 0; r < R; ++r) {
            uint8_t* stA = sU + (r & 1) * L::kRS;  // Phi_Q hi, lo, S hi, lo
            const int nr = min(kRT, F - r * kRT);
            {
                float o[32];
                fe::Eval<D, N, true>::block(r * 2 + half, sQ + kmaj(row, 0, L::kSboD), qc, n, F, tau, o);
                if (row >= nq) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0.f;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t off = kmaj(row, half * 4 + i, kSbo64);
                    store_split8(o + 8 * i, stA + off, stA + L::kA + off);
                }
            }
            if (!wait_bar(&bar_st, r & 1)) bad = true;
            __syncthreads();  // staged z visible
            for (int u = tid; u < kRT * 10; u += kThreads) {
                const int j = u / 10, gq = u % 10;
                float x8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (j < nr && !bad) {
                    if (gq < 8) {
                        const float4 a = *reinterpret_cast<const float4*>(stg + j * kDV + gq * 8);
                        const float4 b = *reinterpret_cast<const float4*>(stg + j * kDV + gq * 8 + 4);
                        x8[0] = a.x; x8[1] = a.y; x8[2] = a.z; x8[3] = a.w;
                        x8[4] = b.x; x8[5] = b.y; x8[6] = b.z; x8[7] = b.w;
                    } else if (gq == 8) {
                        x8[0] = stg_z[j];
                    }
                }
                const uint32_t off = mnmaj(j, gq, kLboNV);
                store_split8(x8, stA + 2 * L::kA + off, stA + 2 * L::kA + L::kB + off);
            }
            if (publish(bad)) {
                bad = true;
                break;
            }
            if (tid == 0) {
                const uint32_t id = idesc_bf16(kQ, kNV, 0, 1);
#pragma unroll
                for (int ks = 0; ks < kRT / 16; ++ks) {
                    const uint64_t ah = smem_desc(stA + ks * 256, 128, kSbo64);
                    const uint64_t al = smem_desc(stA + L::kA + ks * 256, 128, kSbo64);
                    const uint64_t bh_ = smem_desc(stA + 2 * L::kA + ks * 2 * kLboNV, kLboNV, 128);
                    const uint64_t bl_ = smem_desc(stA + 2 * L::kA + L::kB + ks * 2 * kLboNV, kLboNV, 128);
                    mma_bf16(tO, ah, bh_, id, 1u);
                    mma_bf16(tO, ah, bl_, id, 1u);
                    mma_bf16(tO, al, bh_, id, 1u);
                }
                mma_commit(&bar_ro[r & 1]);
            }
            ro_issued = r + 1;
            if (r + 1 < R) fetch_s(r + 1);  // the staging was consumed before the barrier above
            // stage (r + 1) & 1 was last read by the MMAs of tile r - 1
            if (r >= 1 && !wait_bar(&bar_ro[(r - 1) & 1], ((r - 1) >> 1) & 1)) bad = true;
        }
        if (!bad && ro_issued > 0 && !wait_bar(&bar_ro[(ro_issued - 1) & 1], ((ro_issued - 1) >> 1) & 1))
            bad = true;
    }
    bad = __syncthreads_or(bad) != 0;
    fence_after_sync();

    // ------------------------------------------------ epilogue
    if (!bad) {
        float o[32], dn[16];
        tmem_ld32(tO + lane_off + half * 32, o);
        tmem_ld16(tO + lane_off + kDV, dn);
        tmem_ld_wait();
        if (row < nq) {
            const float rcp = __frcp_rn(dn[0]);
            float4* dst = reinterpret_cast<float4*>(out + ((int64_t)bh * Ntok + q0 + row) * kDV + half * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(o[4 * i] * rcp, o[4 * i + 1] * rcp, o[4 * i + 2] * rcp, o[4 * i + 3] * rcp);
        }
    } else {
        if (tid == 0) atomicOr(err, kErrPrefillPipe);
        // bounded waits for work that may still be in flight
        wait_bar(&bar_pv[(T - 1) & 1], ((T - 1) >> 1) & 1);
        if (ro_issued > 0) wait_bar(&bar_ro[(ro_issued - 1) & 1], ((ro_issued - 1) >> 1) & 1);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tslot, 256);
    }
}

constexpr int kMaxDevices = 64;

}  // namespace

namespace tcf {

template <int D, int N>
int run(const bf16* q, const bf16* k, const bf16* v, float* out, const float* state_in, float* state_out, int BH,
        int Ntok, int n, float tau, int64_t F, int64_t stride, unsigned int* err, cudaStream_t stream) {
    static std::once_flag once[kMaxDevices];
    static cudaError_t res[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TAYLOR_ERR_CUDA;
    std::call_once(once[dev], [&]() {
        res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_state_kernel<D, N>),
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StateSmem<D>::kBytes);
        if (res[dev] == cudaSuccess)
            res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_out_kernel<D, N>),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OutSmem<D>::kBytes);
    });
    if (res[dev] != cudaSuccess) return TAYLOR_ERR_CUDA;

    // group size: about F tokens (the pairwise work of a query tile then
    // stays below its read-out work), in [128, 2048], no larger than needed
    int G = 128;
    while (G < 2048 && 2 * (int64_t)G <= F) G *= 2;
    while (G > 128 && G / 2 >= Ntok) G /= 2;
    const int NG = (Ntok + G - 1) / G;
    const int NFT = (int)((F + kFT - 1) / kFT);
    const bool need_ws = NG > 1 || state_in || state_out;
    float* Wb = nullptr;
    if (need_ws) {
        if (workspace_alloc(reinterpret_cast<void**>(&Wb), (size_t)BH * NG * stride * sizeof(float), stream) !=
            cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_OUT_OF_MEMORY;
        }
    }
    cudaError_t e = cudaSuccess;
    if (need_ws) {
        TA_TIMED(stream, "tcf_state_kernel",
                 tcf_state_kernel<D, N><<<dim3(NG, NFT, BH), kThreads, StateSmem<D>::kBytes, stream>>>(
                     k, v, Wb, Ntok, n, (int)F, stride, G, NG, err));
        e = cudaGetLastError();
        if (e == cudaSuccess)
            e = launch_state_scan(Wb, state_in, state_out, BH, NG, stride, F * (kDV + 1), stream, true);
    }
    if (e == cudaSuccess) {
        const int NQ = (Ntok + kQ - 1) / kQ;
        TA_TIMED(stream, "tcf_out_kernel",
                 e = launch_maybe_pdl(tcf_out_kernel<D, N>, dim3(NQ, BH), dim3(kThreads), OutSmem<D>::kBytes, stream,
                                      need_ws, q, k, v, (const float*)Wb, out, Ntok, n, tau, (int)F, stride, G, NG,
                                      state_in != nullptr ? 1 : 0, err));
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    if (Wb) {
        const cudaError_t e2 = workspace_free(Wb, stream);
        if (e == cudaSuccess) e = e2;
    }
    if (e == cudaSuccess) return TAYLOR_OK;
    return e == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
}

}  // namespace tcf
}  // namespace tc
}  // namespace ta
