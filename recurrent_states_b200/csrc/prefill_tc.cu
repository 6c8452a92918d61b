// Chunked causal prefill on the sm_100a tensor cores (tcgen05, TMEM), for
// d_k = 16, n <= 3 (F <= 153, padded to 160) and d_v = 64 with bf16 inputs.
//
// Method (arXiv 2610.20637, abstract): the kernel is an inner product of
// packed tensor powers, so the causal history is the state
// S = sum_j phi(k_j) [v_j | 1]^T, and states are additive across chunks, so
// prefill is a scan.  With chunks of C = 128 tokens:
//   1. tc_chunk_state:  dS_c = Phi_K,c^T [V_c | 1]           (tensor cores)
//   2. scan:            S_<c = sum_{c' < c} dS_c', final state  (CUDA cores)
//   3. tc_chunk_out:    Y_c = (poly(tau Q_c K_c^T) (.) causal mask) [V_c | 1]
//                             + (c (.) Phi_Q,c) S_<c,   o = Y[:, :64] / Y[:, 64]
// Every contraction runs as tcgen05.mma (bf16 operands in shared memory, fp32
// accumulators in TMEM).  bf16 holds 8 significant bits, which alone would
// cost ~4e-3 in the outputs; each operand produced in fp32 (Phi_Q, Phi_K, the
// pairwise weights P and the carried state S) is therefore split into
// hi = bf16(x) and lo = bf16(x - hi) and contracted as hi*hi' + hi*lo' +
// lo*hi' (or hi*B + lo*B when B is an exact bf16 input), which keeps about 16
// significant bits with fp32 accumulation and bf16's full exponent range.
// The normaliser rides along as column 64 of [V | 1 | 0...] (N = 80), so the
// denominator comes out of the same MMAs as the numerator.
//
// The feature map for d_k = 16 is evaluated in closed form with compile-time
// indices: phi = [1, x_i, w_ab x_a x_b (a <= b)], w = sqrt(2) for a < b, 1 for
// a = b, times tau^m/m! on the query side; degrees >= n are zeroed.
#include <algorithm>
#include <mutex>
#include <type_traits>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "prefill_tc.h"
#include "phase.cuh"
#include "phi16.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace ta {
namespace tc {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kC = 128;       // tokens per chunk (MMA M)
constexpr int kD = 16;        // d_k
constexpr int kDV = 64;       // d_v
constexpr int kNV = 80;       // columns of [V | 1 | 0 ...]  (MMA N)
constexpr int kFP = 160;      // features padded to a multiple of 16
constexpr int kThreads = 256;
constexpr uint32_t kWaitPolls = 1u << 24;

// Shared-memory layouts (bytes).  K-major operands use LBO = 128; MN-major
// operands use SBO = 128 (see tcgen05.cuh).
constexpr uint32_t kSboQK = 2 * 128;                 // Q, K: [128][16] K-major
constexpr uint32_t kLboV1 = (kNV / 8) * 128;         // [V|1]: [K=128 keys][80] MN-major
constexpr uint32_t kSboP = (kC / 8) * 128;           // P: [128][128] K-major
constexpr uint32_t kSboPhiQ = (kFP / 8) * 128;       // Phi_Q: [128][160] K-major
constexpr uint32_t kLboS = (2 * kNV / 8) * 128;      // S: [K=160][hi 80 | lo 80] MN-major
constexpr uint32_t kLboVT = 16 * 128;                // [V|1|0]^T: [M=128 rows][K=128 tokens] MN-major
constexpr uint32_t kLboPhiK = (kFP / 8) * 128;       // Phi_K: [K=128 tokens][N=160] MN-major

// chunk_out
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kC * kD * 2;
constexpr uint32_t kOffV1 = kOffK + kC * kD * 2;
constexpr uint32_t kOffPh = kOffV1 + kC * kNV * 2;
constexpr uint32_t kOffPl = kOffPh + kC * kC * 2;
constexpr uint32_t kOffQh = kOffPl + kC * kC * 2;
constexpr uint32_t kOffQl = kOffQh + kC * kFP * 2;
constexpr uint32_t kOffSh = kOffQl + kC * kFP * 2;
constexpr uint32_t kOffSl = kOffSh + kFP * kNV * 2;
constexpr uint32_t kSmemOut = kOffSl + kFP * kNV * 2;   // 227,328 bytes
// chunk_state (transposed: dS^T = [V|1|0]^T Phi_K, so D has the v column on
// the TMEM lanes and the feature on the TMEM columns)
constexpr uint32_t kOffVT = 0;
constexpr uint32_t kOffBh = kOffVT + 128 * kC * 2;
constexpr uint32_t kOffBl = kOffBh + kC * kFP * 2;
constexpr uint32_t kSmemState = kOffBl + kC * kFP * 2;  // 114,688 bytes: two CTAs per SM

static_assert(kSmemOut <= 232448 - 256, "chunk_out shared memory");


__device__ __forceinline__ void ld_row16(const bf16* p, float (&x)[16]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity) {
    const bool ok = ptx::mbar_wait(bar, parity, kWaitPolls);
    return __syncthreads_and(ok) != 0;
}

// ---------------------------------------------------------------- 1. chunk states
// dS_c^T [128 x 160] = [V_c | 1 | 0]^T [128 x 128 tokens] x Phi_K,c [128 tokens x 160]
// with Phi_K as hi + lo.  Lane c < 64 of D is column c of S_v, lane 64 is z.
// The result is staged in shared memory in the state layout and written with
// one bulk copy.
__global__ void __launch_bounds__(kThreads, 2)
tc_chunk_state_kernel(const bf16* __restrict__ k, const bf16* __restrict__ v, float* __restrict__ W, int N,
                      int n, int F, int64_t stride, int NC, unsigned int* __restrict__ err) {
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb;
    __shared__ uint32_t tslot;
    uint8_t* sVT = sm + kOffVT;
    uint8_t* sBh = sm + kOffBh;
    uint8_t* sBl = sm + kOffBl;
    float* sOut = reinterpret_cast<float*>(sm + kOffBh);  // reused once the MMAs are done

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    TA_PHASE(0, 0, tid == 0);
    const int c = blockIdx.x, bh = blockIdx.y;
    const int64_t t0 = (int64_t)c * kC;
    const int nv = (int)min64(kC, (int64_t)N - t0);
    const int row = (warp & 3) * 32 + lane;
    const int half = warp >> 2;
    const bool valid = row < nv;

    if (tid == 0) {
        ptx::mbar_init(&mb, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tslot, 256);
        tmem_relinquish();
    }

    // token `row`: half its features (one K row of the MN-major B operand)
    // and half its [v | 1 | 0] column (one K column of the MN-major A operand)
    const int64_t tok = (int64_t)bh * N + t0 + row;
    const uint4* vr = reinterpret_cast<const uint4*>(v + tok * kDV) + half * 4;
    uint4 val[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) val[g] = valid ? __ldg(vr + g) : make_uint4(0, 0, 0, 0);
    float x[16];
    if (valid) {
        ld_row16(k + tok * kD, x);
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4*>(sVT + mnmaj(row, half * 4 + g, kLboVT)) = val[g];
    if (half == 1) {
        *reinterpret_cast<uint4*>(sVT + mnmaj(row, 8, kLboVT)) = make_uint4(valid ? 0x3F80u : 0u, 0, 0, 0);
#pragma unroll
        for (int g = 9; g < 16; ++g) *reinterpret_cast<uint4*>(sVT + mnmaj(row, g, kLboVT)) = make_uint4(0, 0, 0, 0);
    }
    const float e0 = valid ? 1.f : 0.f, e1 = n >= 2 ? 1.f : 0.f, e2 = n >= 3 ? 1.f : 0.f;
    auto put = [&](int g, uint4 hi, uint4 lo) {
        *reinterpret_cast<uint4*>(sBh + mnmaj(row, g, kLboPhiK)) = hi;
        *reinterpret_cast<uint4*>(sBl + mnmaj(row, g, kLboPhiK)) = lo;
    };
    if (half == 0) phi16_groups<0, 10>(x, e0, e1, e2, put);
    else phi16_groups<10, 20>(x, e0, e1, e2, put);

    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tslot;
    TA_PHASE(0, 1, tid == 0);
    ptx::pdl_launch_dependents();

    if (tid == 0) {
        const uint32_t id = idesc_bf16(128, kFP, 1, 1);
        // descriptors built once and advanced by constants (16-byte units)
        const uint64_t va = smem_desc(sVT, kLboVT, 128);
        const uint64_t bh_ = smem_desc(sBh, kLboPhiK, 128), bl_ = smem_desc(sBl, kLboPhiK, 128);
#pragma unroll
        for (int ks = 0; ks < kC / 16; ++ks) {
            const uint64_t a = va + (2 * kLboVT / 16) * ks;
            mma_bf16(tbase, a, bh_ + (2 * kLboPhiK / 16) * ks, id, ks > 0 ? 1u : 0u);
            mma_bf16(tbase, a, bl_ + (2 * kLboPhiK / 16) * ks, id, 1u);
        }
        mma_commit(&mb);
    }
    const bool ok = wait_all(&mb, 0);
    fence_after_sync();
    TA_PHASE(0, 2, tid == 0);
    const uint32_t bytes = (uint32_t)(((int64_t)F * (kDV + 1) * 4 + 15) / 16 * 16);
    if (ok) {
        // warps 0,1 (+4,5) hold S_v columns 0..63 on their lanes; warp 2 lane 0
        // (+ warp 6) holds z.  Warp w and w+4 split the 160 feature columns.
        const int wq = warp & 3;
        if (wq < 3) {
            const int col = wq * 32 + lane;
            const uint32_t ta = tbase + ((uint32_t)(wq * 32) << 16);
            const int fb = half * 80;
            float r[5][16];
#pragma unroll
            for (int part = 0; part < 5; ++part) tmem_ld16(ta + fb + part * 16, r[part]);
            tmem_ld_wait();
            if (col < kDV) {
#pragma unroll
                for (int part = 0; part < 5; ++part)
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int f = fb + part * 16 + i;
                        if (f < F) sOut[f * kDV + col] = r[part][i];
                    }
            } else if (col == kDV) {
#pragma unroll
                for (int part = 0; part < 5; ++part)
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int f = fb + part * 16 + i;
                        if (f < F) sOut[F * kDV + f] = r[part][i];
                    }
            }
        }
        if (tid < 4) sOut[F * (kDV + 1) + tid] = 0.f;  // tail of the last 16-byte unit
        ptx::fence_proxy_async_smem();
    } else if (tid == 0) {
        atomicOr(err, kErrPrefillPipe);
    }
    if (!ok) ptx::mbar_wait(&mb, 0, kWaitPolls);
    fence_before_sync();
    __syncthreads();
    TA_PHASE(0, 3, tid == 0);
    if (ok && tid == 0) {
        ptx::bulk_s2g(W + ((int64_t)bh * NC + c) * stride, sOut, bytes);
        ptx::bulk_commit();
        ptx::bulk_wait_read_all();
    }
    TA_PHASE(0, 4, tid == 0);
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, 256);
    }
}

// ---------------------------------------------------------------- 3. chunk outputs
// Warps 0-7 stage operands, build Phi_Q, P and S_<c, and run the epilogue;
// warp 8 allocates TMEM and issues every MMA, driven by mbarriers that the
// other warps arrive on.  Everything that does not depend on the carried
// state (the pairwise part and Phi_Q) comes first, so that with programmatic
// dependent launch it overlaps the scan that produces S_<c.
constexpr int kOutThreads = kThreads + 32;
constexpr int kSUnits = kFP * 8 / kThreads;  // 8-column units of S_v per thread (5)

__global__ void __launch_bounds__(kOutThreads, 1)
tc_chunk_out_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                    const float* __restrict__ W, float* __restrict__ out, int N, int n, float tau, int F,
                    int64_t stride, int NC, int carried, int cpc, unsigned int* __restrict__ err) {
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb_s, mb_o, bar_qk, bar_p, bar_ops;
    __shared__ uint32_t tslot;
    __shared__ int mma_fail;
    uint8_t* sQ = sm + kOffQ;
    uint8_t* sK = sm + kOffK;
    uint8_t* sV1 = sm + kOffV1;
    uint8_t* sPh = sm + kOffPh;
    uint8_t* sPl = sm + kOffPl;
    uint8_t* sQh = sm + kOffQh;
    uint8_t* sQl = sm + kOffQl;
    uint8_t* sS = sm + kOffSh;  // S hi in column groups 0..9, lo in 10..19 (the Sh and Sl space)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y;
    TA_PHASE(1, 0, tid == 0);
    TA_PHASE(2, warp, lane == 0);

    if (tid == 0) {
        ptx::mbar_init(&mb_s, 1);
        ptx::mbar_init(&mb_o, 1);
        ptx::mbar_init(&bar_qk, kThreads);
        ptx::mbar_init(&bar_p, kThreads);
        ptx::mbar_init(&bar_ops, kThreads);
        mma_fail = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tslot;
    const uint32_t tA = tbase;          // scores, columns [0, 128)
    // O in columns [128, 288): [0, 80) takes P[V|1|0] + Phi_Q,hi S_hi + Phi_Q,lo S_hi,
    // [80, 160) Phi_Q,hi S_lo (the read-out's hi operand meets [S_hi | S_lo] in one N = 160 MMA)
    const uint32_t tO = tbase + 128;
    TA_PHASE(1, 1, tid == 0);

    if (warp == 8) {
        // ------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
          uint32_t ops_ph = 0;  // bar_ops completes a phase only for chunks with a carried state
          for (int x = 0; x < cpc; ++x) {
            const int c = cpc * blockIdx.x + x;
            if (c >= NC) break;
            const uint32_t ph = (uint32_t)x & 1u;
            const bool inter = c > 0 || carried != 0;   // S_<c is non-zero
            // descriptors are built once and advanced by constants (16-byte units)
            const uint32_t id = idesc_bf16(128, kNV, 0, 1);
            const uint32_t id160 = idesc_bf16(128, 2 * kNV, 0, 1);
            bool good = ptx::mbar_wait(&bar_qk, ph, kWaitPolls);
            fence_after_sync();
            if (good)
                mma_bf16(tA, smem_desc(sQ, 128, kSboQK), smem_desc(sK, 128, kSboQK), idesc_bf16(128, 128, 0, 0), 0u);
            mma_commit(&mb_s);
            if (good) {
                good = ptx::mbar_wait(&bar_p, ph, kWaitPolls);
                fence_after_sync();
                TA_PHASE(1, 11, true);
                if (good) {
                    const uint64_t bv = smem_desc(sV1, kLboV1, 128);
                    const uint64_t ph = smem_desc(sPh, 128, kSboP), pl = smem_desc(sPl, 128, kSboP);
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks) {
                        const uint64_t b = bv + (2 * kLboV1 / 16) * ks;
                        mma_bf16(tO, ph + 16 * ks, b, id, ks > 0 ? 1u : 0u);
                        mma_bf16(tO, pl + 16 * ks, b, id, 1u);
                    }
                }
            }
            if (good && inter) {
                good = ptx::mbar_wait(&bar_ops, ops_ph, kWaitPolls);
                ops_ph ^= 1u;
                fence_after_sync();
                TA_PHASE(1, 12, true);
                if (good) {
                    const uint64_t ah = smem_desc(sQh, 128, kSboPhiQ), al = smem_desc(sQl, 128, kSboPhiQ);
                    const uint64_t bs = smem_desc(sS, kLboS, 128);
#pragma unroll
                    for (int ks = 0; ks < kFP / 16; ++ks) {
                        const uint64_t b = bs + (2 * kLboS / 16) * ks;
                        mma_bf16(tO, ah + 16 * ks, b, id160, 1u);
                        mma_bf16(tO, al + 16 * ks, b, id, 1u);
                    }
                }
            }
            if (!good) {
                mma_fail = 1;
                atomicOr(err, kErrPrefillPipe);
            }
            mma_commit(&mb_o);  // tracks every MMA issued, also on the error path
            TA_PHASE(1, 13, true);
          }
        }
    } else {
        // ------------------------------------------------ operands and epilogue
        const int row = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        for (int x = 0; x < cpc; ++x) {
        const int c = cpc * blockIdx.x + x;
        if (c >= NC) break;
        const uint32_t ph = (uint32_t)x & 1u;
        const int64_t t0 = (int64_t)c * kC;
        const int nv = (int)min64(kC, (int64_t)N - t0);
        const bool inter = c > 0 || carried != 0;   // S_<c is non-zero
        const bool valid = row < nv;
        const int64_t tok = (int64_t)bh * N + t0 + row;

        // q, k rows (K-major [128][16]); half of [v | 1 | 0] (MN-major [K=128][80])
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
        if (valid) {
            const uint4* qr = reinterpret_cast<const uint4*>(q + tok * kD);
            q0 = __ldg(qr);
            q1 = __ldg(qr + 1);
        }
        const uint4* vr = reinterpret_cast<const uint4*>(v + tok * kDV) + half * 4;
        uint4 val[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) val[g] = valid ? __ldg(vr + g) : make_uint4(0, 0, 0, 0);
        if (half == 0) {
            uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0;
            if (valid) {
                const uint4* kr = reinterpret_cast<const uint4*>(k + tok * kD);
                k0 = __ldg(kr);
                k1 = __ldg(kr + 1);
            }
            *reinterpret_cast<uint4*>(sQ + kmaj(row, 0, kSboQK)) = q0;
            *reinterpret_cast<uint4*>(sQ + kmaj(row, 1, kSboQK)) = q1;
            *reinterpret_cast<uint4*>(sK + kmaj(row, 0, kSboQK)) = k0;
            *reinterpret_cast<uint4*>(sK + kmaj(row, 1, kSboQK)) = k1;
        } else {
            *reinterpret_cast<uint4*>(sV1 + mnmaj(row, 8, kLboV1)) = make_uint4(valid ? 0x3F80u : 0u, 0, 0, 0);
            *reinterpret_cast<uint4*>(sV1 + mnmaj(row, 9, kLboV1)) = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4*>(sV1 + mnmaj(row, half * 4 + g, kLboV1)) = val[g];
        ptx::fence_proxy_async_smem();
        fence_before_sync();  // the previous chunk's TMEM loads, before its accumulators are rewritten
        ptx::mbar_arrive(&bar_qk);
        TA_PHASE(1, 2, tid == 0);

        // half of Phi_Q for token `row` while the scores are computed
        if (inter) {
            float x[16];
            const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                x[2 * i] = __uint_as_float(w[i] << 16);
                x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
            const float e1 = n >= 2 ? tau : 0.f, e2 = n >= 3 ? 0.5f * tau * tau : 0.f;
            auto put = [&](int g, uint4 hi, uint4 lo) {
                *reinterpret_cast<uint4*>(sQh + kmaj(row, g, kSboPhiQ)) = hi;
                *reinterpret_cast<uint4*>(sQl + kmaj(row, g, kSboPhiQ)) = lo;
            };
            if (half == 0) phi16_groups<0, 10>(x, valid ? 1.f : 0.f, e1, e2, put);
            else phi16_groups<10, 20>(x, valid ? 1.f : 0.f, e1, e2, put);
        }
        TA_PHASE(1, 3, tid == 0);

        // pairwise weights P = poly(tau q.k) under the causal mask, hi/lo, K-major
        bool ok = ptx::mbar_wait(&mb_s, ph, kWaitPolls);
        fence_after_sync();
        TA_PHASE(1, 4, tid == 0);
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        {
            float s0[32], s1[32];
            tmem_ld32(tA + lane_off + half * 64, s0);
            tmem_ld32(tA + lane_off + half * 64 + 32, s1);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = g * 8 + e;
                    const int key = half * 64 + j;
                    const float sc = j < 32 ? s0[j] : s1[j - 32];
                    const float xx = tau * sc;
                    float w = 1.f;
                    if (n >= 3) w = 1.f + xx * (1.f + 0.5f * xx);
                    else if (n == 2) w = 1.f + xx;
                    p[e] = (valid && key <= row) ? w : 0.f;
                }
                uint4 hi, lo;
                split8(p, hi, lo);
                const int kg = half * 8 + g;
                *reinterpret_cast<uint4*>(sPh + kmaj(row, kg, kSboP)) = hi;
                *reinterpret_cast<uint4*>(sPl + kmaj(row, kg, kSboP)) = lo;
            }
        }
        ptx::fence_proxy_async_smem();
        fence_before_sync();
        ptx::mbar_arrive(&bar_p);
        TA_PHASE(1, 5, tid == 0);

        // the carried state S_<c: produced by the previous grid
        if (inter) {
            ptx::pdl_wait_primary();
            TA_PHASE(1, 6, tid == 0);
            const float* Sg = W + ((int64_t)bh * NC + c) * stride;
            float4 sa[kSUnits], sb[kSUnits];
#pragma unroll
            for (int i = 0; i < kSUnits; ++i) {
                const int u = tid + i * kThreads, f = u >> 3, g = u & 7;
                if (f < F) {
                    sa[i] = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + g * 8));
                    sb[i] = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + g * 8) + 1);
                } else {
                    sa[i] = sb[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            const float zf = (tid < kFP && tid < F) ? __ldg(Sg + (int64_t)F * kDV + tid) : 0.f;
#pragma unroll
            for (int i = 0; i < kSUnits; ++i) {
                const int u = tid + i * kThreads, f = u >> 3, g = u & 7;
                const float xs[8] = {sa[i].x, sa[i].y, sa[i].z, sa[i].w, sb[i].x, sb[i].y, sb[i].z, sb[i].w};
                uint4 hi, lo;
                split8(xs, hi, lo);
                *reinterpret_cast<uint4*>(sS + mnmaj(f, g, kLboS)) = hi;
                *reinterpret_cast<uint4*>(sS + mnmaj(f, 10 + g, kLboS)) = lo;
            }
            if (tid < kFP) {
                const float xs[8] = {zf, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint4 hi, lo;
                split8(xs, hi, lo);
                *reinterpret_cast<uint4*>(sS + mnmaj(tid, 8, kLboS)) = hi;
                *reinterpret_cast<uint4*>(sS + mnmaj(tid, 18, kLboS)) = lo;
                *reinterpret_cast<uint4*>(sS + mnmaj(tid, 9, kLboS)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sS + mnmaj(tid, 19, kLboS)) = make_uint4(0, 0, 0, 0);
            }
            // O columns 80..159 start at zero: the read-out MMAs into them accumulate
            if (half == 0) {
                uint32_t z[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) z[i] = 0;
                const uint32_t lo_ = (uint32_t)((warp & 3) * 32) << 16;
                tmem_st32(tO + lo_ + 80, z);
                tmem_st32(tO + lo_ + 112, z);
                tmem_st16(tO + lo_ + 144, *reinterpret_cast<uint32_t(*)[16]>(z));
                tmem_st_wait();
            }
            fence_before_sync();
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bar_ops);
            TA_PHASE(1, 7, tid == 0);
        }

        // epilogue: o = numerator * (1 / denominator)
        const bool done = ptx::mbar_wait(&mb_o, ph, kWaitPolls);
        fence_after_sync();
        TA_PHASE(1, 8, tid == 0);
        ok = ok && done && mma_fail == 0;
        if (ok) {
            float o[32], dn[16];
            tmem_ld32(tO + lane_off + half * 32, o);
            tmem_ld16(tO + lane_off + kDV, dn);
            tmem_ld_wait();
            float d2 = 0.f;
            if (inter) {
                float o2[32];
                tmem_ld32(tO + lane_off + kNV + half * 32, o2);
                d2 = tmem_ld1(tO + lane_off + kNV + kDV);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] += o2[i];
            }
            if (valid) {
                const float r = __frcp_rn(dn[0] + d2);
                float4* dst = reinterpret_cast<float4*>(out + tok * kDV + half * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dst[i] = make_float4(o[4 * i] * r, o[4 * i + 1] * r, o[4 * i + 2] * r, o[4 * i + 3] * r);
            }
        } else {
            if (tid == 0) atomicOr(err, kErrPrefillPipe);
            if (!done) ptx::mbar_wait(&mb_o, ph, kWaitPolls);  // one more bound for MMAs in flight
        }
        TA_PHASE(1, 9, tid == 0);
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 8) {
        fence_after_sync();
        tmem_dealloc(tbase, 512);
    }
    TA_PHASE(1, 14, tid == 0);
}

// ---------------------------------------------------------------- 3'. centred outputs
// Output kernel of the mean-centred softmax expansion (Su Jianlin's note on the
// Taylor expansions of logsumexp and softmax, kexue.fm translation 11814,
// sections "Calculating the Gradient" and "Linear Attention") on the tensor
// cores, over the n = 3 chunk states of tc_chunk_state (their degree-0, 1 and 2
// rows hold every prefix sum the expansion needs).  For query i the three
// read-outs R_m = sum_{j <= i} (q_i . k_j)^m [v_j | 1] (no tau, no 1/m!) go to
// three TMEM accumulators:
//   pairwise   P_0 = mask (exact in bf16, shared memory), P_1 = s, P_2 = s^2
//              (s = q_i . k_j, hi/lo, written over the scores in TMEM), each
//              times [V | 1 | 0];
//   carried    phi_m(q) S_<c,m, with the features laid out so that each degree
//              starts a K step of 16: feature 0 at row 0 (rows 1..15 zero), the
//              16 of degree 1 at rows 16..31, the 136 of degree 2 at rows
//              32..167 (168..175 zero).
// Then, per column,
//   n = R_0[z], V = R_0[v], qkbar = R_1[z] / n,
//   sum a v   = tau (R_1[v] - qkbar V),
//   sum a^2 v = tau^2 (R_2[v] - 2 qkbar R_1[v] + qkbar^2 V),
//   sum a^2   = tau^2 (R_2[z] - n qkbar^2),
//   o = V/n + (sum a v)/n  [+ (sum a^2 v - (sum a^2) V/n) / (2n) at order 2].
constexpr int kFC = 176;                          // features, degree-aligned
constexpr uint32_t kSboPhiQC = (kFC / 8) * 128;   // Phi_Q: [128][176] K-major
constexpr uint32_t kCOffQ = 0;
constexpr uint32_t kCOffK = kCOffQ + kC * kD * 2;
constexpr uint32_t kCOffV1 = kCOffK + kC * kD * 2;
constexpr uint32_t kCOffP0 = kCOffV1 + kC * kNV * 2;
constexpr uint32_t kCOffQh = kCOffP0 + kC * kC * 2;
constexpr uint32_t kCOffQl = kCOffQh + kC * kFC * 2;
constexpr uint32_t kCOffS = kCOffQl + kC * kFC * 2;
constexpr uint32_t kSmemCentred = kCOffS + kFC * 2 * kNV * 2;  // 207,872 bytes
static_assert(kSmemCentred <= 232448 - 256, "centred chunk_out shared memory");
// TMEM: scores, then P_1 over them [0, 128); R_0, R_1, R_2 [128, 368); P_2 [368, 496)
constexpr uint32_t kCR0 = 128, kCP2 = 368;
// chunks per CTA, one after the other on the same operand space and TMEM (the
// main workload's 256 chunks then fit one wave, and the second chunk runs on
// fetched code)
constexpr int kCentredChunks = 2;

// padded row of packed feature f (d_k 16, n 3): degree 0 at 0, degrees 1, 2 from 16
__device__ __forceinline__ int centred_row(int f) { return f == 0 ? 0 : f + 15; }

__global__ void __launch_bounds__(kOutThreads, 1)
tc_centred_chunk_out_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
                            const float* __restrict__ W, float* __restrict__ out, int N, int order, float tau,
                            int F, int64_t stride, int NC, int carried, unsigned int* __restrict__ err) {
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb_s, mb_o, bar_qk, bar_p, bar_ops;
    __shared__ uint32_t tslot;
    __shared__ int mma_fail;
    uint8_t* sQ = sm + kCOffQ;
    uint8_t* sK = sm + kCOffK;
    uint8_t* sV1 = sm + kCOffV1;
    uint8_t* sP0 = sm + kCOffP0;
    uint8_t* sQh = sm + kCOffQh;
    uint8_t* sQl = sm + kCOffQl;
    uint8_t* sS = sm + kCOffS;  // [176 rows][S hi in column groups 0..9 | lo in 10..19]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.y;
    const bool second = order >= 2;

    if (tid == 0) {
        ptx::mbar_init(&mb_s, 1);
        ptx::mbar_init(&mb_o, 1);
        ptx::mbar_init(&bar_qk, kThreads);
        ptx::mbar_init(&bar_p, kThreads);
        ptx::mbar_init(&bar_ops, kThreads);
        mma_fail = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tslot;
    const uint32_t tA = tbase;  // scores, then P_1

    if (warp == 8) {
        // ------------------------------------------------ MMA issue (one thread)
        if (lane == 0) {
          uint32_t ops_ph = 0;  // bar_ops completes a phase only for chunks with a carried state
          for (int x = 0; x < kCentredChunks; ++x) {
            const int c = kCentredChunks * blockIdx.x + x;
            if (c >= NC) break;
            const uint32_t ph = (uint32_t)x & 1u;
            const bool inter = c > 0 || carried != 0;   // S_<c is non-zero
            const uint32_t id = idesc_bf16(128, kNV, 0, 1);
            const uint64_t bv = smem_desc(sV1, kLboV1, 128);
            bool good = ptx::mbar_wait(&bar_qk, ph, kWaitPolls);
            fence_after_sync();
            if (good) {
                mma_bf16(tA, smem_desc(sQ, 128, kSboQK), smem_desc(sK, 128, kSboQK), idesc_bf16(128, 128, 0, 0), 0u);
                mma_commit(&mb_s);
                // R_0 = P_0 [V | 1 | 0] needs no scores
                const uint64_t p0 = smem_desc(sP0, 128, kSboP);
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks)
                    mma_bf16(tbase + kCR0, p0 + 16 * ks, bv + (2 * kLboV1 / 16) * ks, id, ks > 0 ? 1u : 0u);
            } else {
                mma_commit(&mb_s);
            }
            if (good) {
                good = ptx::mbar_wait(&bar_p, ph, kWaitPolls);
                fence_after_sync();
                if (good) {
                    // R_1 = P_1 [V | 1 | 0], R_2 = P_2 [V | 1 | 0]; P of keys 16 ks .. 16 ks + 15:
                    // hi words at 32 (ks / 2) + 8 (ks % 2), lo 16 further
#pragma unroll
                    for (int ks = 0; ks < kC / 16; ++ks) {
                        const uint64_t b = bv + (2 * kLboV1 / 16) * ks;
                        const uint32_t a = 32 * (ks >> 1) + 8 * (ks & 1);
                        mma_bf16_ts(tbase + kCR0 + 80, tA + a, b, id, ks > 0 ? 1u : 0u);
                        mma_bf16_ts(tbase + kCR0 + 80, tA + a + 16, b, id, 1u);
                        if (second) {
                            mma_bf16_ts(tbase + kCR0 + 160, tbase + kCP2 + a, b, id, ks > 0 ? 1u : 0u);
                            mma_bf16_ts(tbase + kCR0 + 160, tbase + kCP2 + a + 16, b, id, 1u);
                        }
                    }
                }
            }
            if (good && inter) {
                good = ptx::mbar_wait(&bar_ops, ops_ph, kWaitPolls);
                ops_ph ^= 1u;
                fence_after_sync();
                if (good) {
                    // K step 0 -> R_0 (Phi_Q of feature 0 is exact: no lo term),
                    // step 1 -> R_1, steps 2..10 -> R_2
                    const uint64_t ah = smem_desc(sQh, 128, kSboPhiQC), al = smem_desc(sQl, 128, kSboPhiQC);
                    const uint64_t sh = smem_desc(sS, kLboS, 128), sl = smem_desc(sS + 10 * 128, kLboS, 128);
                    const int nks = second ? kFC / 16 : 2;
#pragma unroll 1
                    for (int ks = 0; ks < nks; ++ks) {
                        const uint32_t d = tbase + kCR0 + 80 * min(ks, 2);
                        const uint64_t bh_ = sh + (2 * kLboS / 16) * ks, bl_ = sl + (2 * kLboS / 16) * ks;
                        mma_bf16(d, ah + 16 * ks, bh_, id, 1u);
                        mma_bf16(d, ah + 16 * ks, bl_, id, 1u);
                        if (ks > 0) mma_bf16(d, al + 16 * ks, bh_, id, 1u);
                    }
                }
            }
            if (!good) {
                mma_fail = 1;
                atomicOr(err, kErrPrefillPipe);
            }
            mma_commit(&mb_o);  // tracks every MMA issued, also on the error path
          }
        }
    } else {
        // ------------------------------------------------ operands and epilogue
        const int row = (warp & 3) * 32 + lane;
        const int half = warp >> 2;
        for (int x = 0; x < kCentredChunks; ++x) {
        const int c = kCentredChunks * blockIdx.x + x;
        if (c >= NC) break;
        const uint32_t ph = (uint32_t)x & 1u;
        const int64_t t0 = (int64_t)c * kC;
        const int nv = (int)min64(kC, (int64_t)N - t0);
        const bool inter = c > 0 || carried != 0;   // S_<c is non-zero
        const bool valid = row < nv;
        const int64_t tok = (int64_t)bh * N + t0 + row;

        // q, k rows (K-major [128][16]); half of [v | 1 | 0] (MN-major [K=128][80]);
        // row `row` of P_0, keys [64 half, 64 half + 64)
        uint4 q0 = make_uint4(0, 0, 0, 0), q1 = q0;
        if (valid) {
            const uint4* qr = reinterpret_cast<const uint4*>(q + tok * kD);
            q0 = __ldg(qr);
            q1 = __ldg(qr + 1);
        }
        const uint4* vr = reinterpret_cast<const uint4*>(v + tok * kDV) + half * 4;
        uint4 val[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) val[g] = valid ? __ldg(vr + g) : make_uint4(0, 0, 0, 0);
        if (half == 0) {
            uint4 k0 = make_uint4(0, 0, 0, 0), k1 = k0;
            if (valid) {
                const uint4* kr = reinterpret_cast<const uint4*>(k + tok * kD);
                k0 = __ldg(kr);
                k1 = __ldg(kr + 1);
            }
            *reinterpret_cast<uint4*>(sQ + kmaj(row, 0, kSboQK)) = q0;
            *reinterpret_cast<uint4*>(sQ + kmaj(row, 1, kSboQK)) = q1;
            *reinterpret_cast<uint4*>(sK + kmaj(row, 0, kSboQK)) = k0;
            *reinterpret_cast<uint4*>(sK + kmaj(row, 1, kSboQK)) = k1;
        } else {
            *reinterpret_cast<uint4*>(sV1 + mnmaj(row, 8, kLboV1)) = make_uint4(valid ? 0x3F80u : 0u, 0, 0, 0);
            *reinterpret_cast<uint4*>(sV1 + mnmaj(row, 9, kLboV1)) = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4*>(sV1 + mnmaj(row, half * 4 + g, kLboV1)) = val[g];
        // (the causal mask is the same for every chunk)
#pragma unroll
        for (int g = 0; g < 8 && x == 0; ++g) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int key = half * 64 + g * 8 + 2 * e;
                w[e] = (key <= row ? 0x3F80u : 0u) | (key + 1 <= row ? 0x3F800000u : 0u);
            }
            *reinterpret_cast<uint4*>(sP0 + kmaj(row, half * 8 + g, kSboP)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        ptx::fence_proxy_async_smem();
        fence_before_sync();  // the previous chunk's TMEM loads, before its accumulators are rewritten
        ptx::mbar_arrive(&bar_qk);

        // phi(q) for token `row` (multinomial weights only), degree-aligned:
        // half 0 K steps 0..5, half 1 K steps 6..10
        if (inter) {
            float x[16];
            const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                x[2 * i] = __uint_as_float(w[i] << 16);
                x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
            const float e0 = valid ? 1.f : 0.f;
            auto step = [&](auto kb) {
                constexpr int KS = decltype(kb)::value;
                float o[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) o[i] = 0.f;
                if (KS == 0) {
                    o[0] = e0;
                } else {
                    // packed features 16 KS - 15 .. 16 KS (feature 160 and beyond stay zero)
                    constexpr int F0 = 16 * KS - 15, F1 = F0 + 16 > 160 ? 160 : F0 + 16;
                    float t[F1 - F0];
                    phi16_range<F0, F1>(x, e0, 1.f, 1.f, t);
#pragma unroll
                    for (int i = 0; i < F1 - F0; ++i) o[i] = t[i];
                }
                uint4 hi0, lo0, hi1, lo1;
                split8(o, hi0, lo0);
                split8(o + 8, hi1, lo1);
                *reinterpret_cast<uint4*>(sQh + kmaj(row, 2 * KS, kSboPhiQC)) = hi0;
                *reinterpret_cast<uint4*>(sQh + kmaj(row, 2 * KS + 1, kSboPhiQC)) = hi1;
                *reinterpret_cast<uint4*>(sQl + kmaj(row, 2 * KS, kSboPhiQC)) = lo0;
                *reinterpret_cast<uint4*>(sQl + kmaj(row, 2 * KS + 1, kSboPhiQC)) = lo1;
            };
            if (half == 0) {
                step(std::integral_constant<int, 0>());
                step(std::integral_constant<int, 1>());
                if (second) {
                    step(std::integral_constant<int, 2>());
                    step(std::integral_constant<int, 3>());
                    step(std::integral_constant<int, 4>());
                    step(std::integral_constant<int, 5>());
                }
            } else if (second) {
                step(std::integral_constant<int, 6>());
                step(std::integral_constant<int, 7>());
                step(std::integral_constant<int, 8>());
                step(std::integral_constant<int, 9>());
                step(std::integral_constant<int, 10>());
            }
        }

        // P_1 = s, P_2 = s^2 under the causal mask, hi/lo, into TMEM (P_1 over
        // the scores, each 32-key piece: 16 hi words, then 16 lo words)
        bool ok = ptx::mbar_wait(&mb_s, ph, kWaitPolls);
        fence_after_sync();
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
#pragma unroll
        for (int pc = 0; pc < 2; ++pc) {
            const uint32_t col = lane_off + 64 * half + 32 * pc;
            float s[32];
            tmem_ld32(tA + col, s);
            tmem_ld_wait();
            uint32_t h1[16], l1[16], h2[16], l2[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                float p1[2], p2[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool on = valid && 64 * half + 32 * pc + j + e <= row;
                    p1[e] = on ? s[j + e] : 0.f;
                    p2[e] = p1[e] * p1[e];
                }
                split2(p1[0], p1[1], h1[j >> 1], l1[j >> 1]);
                split2(p2[0], p2[1], h2[j >> 1], l2[j >> 1]);
            }
            tmem_st16(tA + col, h1);
            tmem_st16(tA + col + 16, l1);
            if (second) {
                tmem_st16(tbase + kCP2 + col, h2);
                tmem_st16(tbase + kCP2 + col + 16, l2);
            }
        }
        tmem_st_wait();
        fence_before_sync();
        ptx::mbar_arrive(&bar_p);

        // the carried state S_<c: produced by the previous grid
        if (inter) {
            ptx::pdl_wait_primary();
            const float* Sg = W + ((int64_t)bh * NC + c) * stride;
            float4 sa[kSUnits], sb[kSUnits];
#pragma unroll
            for (int i = 0; i < kSUnits; ++i) {
                const int u = tid + i * kThreads, f = u >> 3, g = u & 7;
                if (f < F) {
                    sa[i] = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + g * 8));
                    sb[i] = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + g * 8) + 1);
                } else {
                    sa[i] = sb[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            const float zf = tid < F ? __ldg(Sg + (int64_t)F * kDV + tid) : 0.f;
#pragma unroll
            for (int i = 0; i < kSUnits; ++i) {
                const int u = tid + i * kThreads, f = u >> 3, g = u & 7;
                if (f < F) {
                    const float xs[8] = {sa[i].x, sa[i].y, sa[i].z, sa[i].w, sb[i].x, sb[i].y, sb[i].z, sb[i].w};
                    uint4 hi, lo;
                    split8(xs, hi, lo);
                    const int r = centred_row(f);
                    *reinterpret_cast<uint4*>(sS + mnmaj(r, g, kLboS)) = hi;
                    *reinterpret_cast<uint4*>(sS + mnmaj(r, 10 + g, kLboS)) = lo;
                }
            }
            if (tid < F) {
                const float xs[8] = {zf, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint4 hi, lo;
                split8(xs, hi, lo);
                const int r = centred_row(tid);
                *reinterpret_cast<uint4*>(sS + mnmaj(r, 8, kLboS)) = hi;
                *reinterpret_cast<uint4*>(sS + mnmaj(r, 18, kLboS)) = lo;
                *reinterpret_cast<uint4*>(sS + mnmaj(r, 9, kLboS)) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(sS + mnmaj(r, 19, kLboS)) = make_uint4(0, 0, 0, 0);
            }
            // the rows no feature maps to: 1..15 and F + 15 .. 175
            const int nzero = 15 + (kFC - (F + 15));
            for (int u = tid; u < nzero * 20; u += kThreads) {
                const int zr = u / 20, g = u % 20;
                const int r = zr < 15 ? 1 + zr : F + 15 + (zr - 15);
                *reinterpret_cast<uint4*>(sS + mnmaj(r, g, kLboS)) = make_uint4(0, 0, 0, 0);
            }
            fence_before_sync();
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&bar_ops);
        }

        // epilogue: the combination of R_0, R_1 (, R_2) per column
        const bool done = ptx::mbar_wait(&mb_o, ph, kWaitPolls);
        fence_after_sync();
        ok = ok && done && mma_fail == 0;
        if (ok) {
            const uint32_t tr = tbase + kCR0 + lane_off;
            const float z0 = tmem_ld1(tr + kDV), z1 = tmem_ld1(tr + 80 + kDV);
            const float z2 = second ? tmem_ld1(tr + 160 + kDV) : 0.f;
            tmem_ld_wait();
            const float nn = z0, qkbar = z1 / nn, t2 = tau * tau;
            const float sum_a2 = t2 * (z2 - nn * qkbar * qkbar);
            // 16 columns at a time
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const uint32_t cc = half * 32 + cb * 16;
                float a0[16], a1[16], a2[16];
                tmem_ld16(tr + cc, a0);
                tmem_ld16(tr + 80 + cc, a1);
                if (second) tmem_ld16(tr + 160 + cc, a2);
                tmem_ld_wait();
                if (valid) {
                    float r[16];
#pragma unroll
                    for (int c2 = 0; c2 < 16; ++c2) {
                        const float V = a0[c2];
                        float xo = V / nn + tau * (a1[c2] - qkbar * V) / nn;
                        if (second) {
                            const float sum_a2v = t2 * (a2[c2] - 2.0f * qkbar * a1[c2] + qkbar * qkbar * V);
                            xo += (sum_a2v - sum_a2 * V / nn) / (2.0f * nn);
                        }
                        r[c2] = xo;
                    }
                    float4* dst = reinterpret_cast<float4*>(out + tok * kDV + cc);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
                }
            }
        } else {
            if (tid == 0) atomicOr(err, kErrPrefillPipe);
            if (!done) ptx::mbar_wait(&mb_o, ph, kWaitPolls);  // one more bound for MMAs in flight
        }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 8) {
        fence_after_sync();
        tmem_dealloc(tbase, 512);
    }
}

constexpr int kMaxDevices = 64;

cudaError_t set_smem_once(const void* fn, int bytes, std::once_flag* once, cudaError_t* res) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        res[dev] = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    });
    return res[dev];
}

}  // namespace

int try_prefill(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau, int64_t F,
                int64_t stride, cudaStream_t stream) {
    if (d != kD || dv != kDV || n > 3 || N <= 0 || BH <= 0) return kNotApplicable;
    unsigned int* err = device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;

    static std::once_flag once_a[kMaxDevices], once_c[kMaxDevices];
    static cudaError_t res_a[kMaxDevices], res_c[kMaxDevices];
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(tc_chunk_state_kernel), (int)kSmemState, once_a, res_a);
    if (e == cudaSuccess)
        e = set_smem_once(reinterpret_cast<const void*>(tc_chunk_out_kernel), (int)kSmemOut, once_c, res_c);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_CUDA;
    }

    const int NC = (N + kC - 1) / kC;
    const size_t ws_bytes = (size_t)BH * NC * stride * sizeof(float);
    float* W = nullptr;
    if (workspace_alloc(reinterpret_cast<void**>(&W), ws_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_OUT_OF_MEMORY;
    }
    const dim3 grid(NC, BH);
    TA_TIMED(stream, "tc_chunk_state_kernel",
             tc_chunk_state_kernel<<<grid, kThreads, kSmemState, stream>>>(k, v, W, N, n, (int)F, stride, NC, err));
    e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_state_scan(W, state_in, state_out, BH, NC, stride, F * (dv + 1), stream, true);
    if (e == cudaSuccess) {
        // up to four chunks a CTA (one after another), so that a call with more
        // chunks than SMs runs in fewer waves and later chunks on fetched code
        int sms = 148;
        int dev = 0;
        if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
            cudaGetLastError();
            sms = 148;
        }
        const int64_t total = (int64_t)NC * BH;
        const int cpc = (int)std::min<int64_t>(4, std::max<int64_t>(1, (total + sms - 1) / sms));
        const dim3 grid_o((NC + cpc - 1) / cpc, BH);
        TA_TIMED(stream, "tc_chunk_out_kernel",
                 e = launch_maybe_pdl(tc_chunk_out_kernel, grid_o, dim3(kOutThreads), kSmemOut, stream, true, q, k, v,
                                      W, out, N, n, tau, (int)F, stride, NC, state_in != nullptr ? 1 : 0, cpc, err));
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    const cudaError_t e2 = workspace_free(W, stream);
    if (e == cudaSuccess) e = e2;
    if (e == cudaSuccess) return TAYLOR_OK;
    return e == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
}

int try_centred_prefill(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                        float* state_out, int BH, int N, int d, int dv, int order, float tau, int64_t F,
                        int64_t stride, cudaStream_t stream) {
    if (d != kD || dv != kDV || F != 153 || N <= 0 || BH <= 0 || (order != 1 && order != 2)) return kNotApplicable;
    unsigned int* err = device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;

    static std::once_flag once_a[kMaxDevices], once_c[kMaxDevices];
    static cudaError_t res_a[kMaxDevices], res_c[kMaxDevices];
    cudaError_t e = set_smem_once(reinterpret_cast<const void*>(tc_chunk_state_kernel), (int)kSmemState, once_a, res_a);
    if (e == cudaSuccess)
        e = set_smem_once(reinterpret_cast<const void*>(tc_centred_chunk_out_kernel), (int)kSmemCentred, once_c,
                          res_c);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_CUDA;
    }

    // the n = 3 chunk states and their exclusive scan, as the Taylor prefill forms them
    const int NC = (N + kC - 1) / kC;
    const size_t ws_bytes = (size_t)BH * NC * stride * sizeof(float);
    float* W = nullptr;
    if (workspace_alloc(reinterpret_cast<void**>(&W), ws_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_OUT_OF_MEMORY;
    }
    const dim3 grid(NC, BH);
    TA_TIMED(stream, "tc_chunk_state_kernel",
             tc_chunk_state_kernel<<<grid, kThreads, kSmemState, stream>>>(k, v, W, N, 3, (int)F, stride, NC, err));
    e = cudaGetLastError();
    if (e == cudaSuccess) e = launch_state_scan(W, nullptr, state_out, BH, NC, stride, F * (dv + 1), stream, true);
    if (e == cudaSuccess) {
        const dim3 grid_o((NC + kCentredChunks - 1) / kCentredChunks, BH);
        TA_TIMED(stream, "tc_centred_chunk_out_kernel",
                 e = launch_maybe_pdl(tc_centred_chunk_out_kernel, grid_o, dim3(kOutThreads), kSmemCentred, stream, true,
                                      q, k, v, (const float*)W, out, N, order, tau, (int)F, stride, NC, 0, err));
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    const cudaError_t e2 = workspace_free(W, stream);
    if (e == cudaSuccess) e = e2;
    if (e == cudaSuccess) return TAYLOR_OK;
    return e == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
}

}  // namespace tc
}  // namespace ta
