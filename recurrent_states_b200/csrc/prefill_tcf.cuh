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
//   2, 3. tcf_scan_pack_kernel: the exclusive scan over groups, each prefix
//      S_<g written straight as 64-feature read-out operand tiles, split
//      into hi/lo bf16 once per group rather than once per query tile;
//   4. tcf_out_kernel (128 queries, head):
//        O = sum over 64-key tiles of the group up to the diagonal of
//              (poly(tau Q K^T) (.) mask) [V|1|0]
//          + sum over 64-feature tiles of (c (.) Phi_Q[:, tile]) S_<g[tile, :],
//        o = O[:, :64] / O[:, 64].
// Operands produced in fp32 (Phi_K, Phi_Q, P and S_<g) are split into hi/lo
// bf16 pairs (about 16 significant bits reach the fp32 accumulators); q, k and
// v are bf16 already.
//
// Both CTA kinds are warp-specialised.  One thread issues TMA tensor loads
// (whole q, k, v rows into the swizzled K-major / MN-major operand layouts,
// zero-filled past the sequence), one thread issues every tcgen05.mma, and two warpgroups of
// CUDA cores evaluate features (or P) for alternate stages, so that the
// loads, the tensor cores and the feature arithmetic of different stages run
// at the same time.  In the output kernel the operands the CUDA cores produce
// (P and Phi_Q, hi/lo) go to TMEM with tcgen05.st and the MMAs read them from
// there (A in TMEM, B in shared memory), which keeps the tensor cores' shared
// memory reads to the B operand: with N = 80 an MMA reading A from shared
// memory as well would need more bytes per cycle than shared memory gives.
// Hand-offs are mbarriers: TMA transaction counts, 128 arrivals from a
// warpgroup, or tcgen05.commit.  Every wait is bounded and a
// failed wait stops the other roles' waits too; a device error bit records it.
#pragma once

#include <cuda.h>

#include <mutex>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "feat_eval.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "phase.cuh"
#include "prefill_tc.h"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tmap.h"

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
constexpr int kCompute = 256; // two warpgroups
constexpr uint32_t kWaitPolls = 1u << 24;

constexpr uint32_t kVAtom = kTok * 128;         // 64 token rows of 64 v columns, 128-byte swizzle (8 KB)
constexpr uint32_t kPhiBytes = kTok * kFT * 2;   // state-stage Phi_K, hi or lo
constexpr uint32_t kLboFT = (kFT / 8) * 128;     // its K-group stride
constexpr uint32_t kLboS = (2 * kNV / 8) * 128;  // K-group stride of a packed S tile
constexpr uint32_t kSTile = kRT * 2 * kNV * 2;   // packed S tile [64 features][hi 80 | lo 80] (20 KB)

__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, volatile int* bad) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitPolls, bad);
}

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
    const uint32_t a = ptx::smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// 64 fp32 values -> hi/lo bf16 pairs, K order, as 32 + 32 words of a TMEM
// A-operand row.
__device__ __forceinline__ void split64_words(const float* x, uint32_t (&hi)[32], uint32_t (&lo)[32]) {
#pragma unroll
    for (int i = 0; i < 32; ++i) split2(x[2 * i], x[2 * i + 1], hi[i], lo[i]);
}

// Eight fp32 values -> hi/lo bf16 chunks stored at two operand addresses.
__device__ __forceinline__ void store_split8(const float* x, uint8_t* hi_dst, uint8_t* lo_dst) {
    uint4 hi, lo;
    split8(x, hi, lo);
    *reinterpret_cast<uint4*>(hi_dst) = hi;
    *reinterpret_cast<uint4*>(lo_dst) = lo;
}

// q and k rows as TMA writes them: K-major operands with D-element rows
// (32, 64 or 128 bytes) under the matching swizzle.
template <int D>
struct RowSw {
    static constexpr uint32_t kRowBytes = D * 2;
    static constexpr uint32_t kLayout = D == 64 ? kSwizzle128 : D == 32 ? kSwizzle64 : kSwizzle32;
    static constexpr uint32_t kSbo = 8 * kRowBytes;
};

// The [v | 1 | 0] operand is MN-major [K = 64 tokens][N = 80] under the
// 128-byte swizzle: atom 0 (columns 0..63) is a slot that TMA fills with v
// rows; atom 1 (columns 64..127, of which the MMA reads 64..79) is one ones
// atom shared by every slot, reached through the descriptor's LBO: column 64
// is 1 and the rest 0, in every token row.
__device__ __forceinline__ void init_ones_atom(uint8_t* atom, int tid, int nthreads) {
    for (int i = tid; i < kTok * 8; i += nthreads) {
        const int k = i >> 3, c = i & 7;
        *reinterpret_cast<uint4*>(atom + k * 128 + ((c ^ (k & 7)) << 4)) = make_uint4(c == 0 ? 0x3F80u : 0u, 0, 0, 0);
    }
}

// ---------------------------------------------------------------- 1. group states
// Shared memory: four Phi_K slots (stage s uses slot s % 4 and belongs to
// warpgroup s & 1), four v slots beside them plus the ones atom, and a
// separate ring of six k-row slots, released as soon as a warpgroup has read
// its rows, so that k loads run several stages ahead of the evaluation.
template <int D>
struct StSm {
    static constexpr int kSlots = 2;
    static constexpr int kKSlots = 2;
    static constexpr uint32_t kK = kTok * D * 2;  // k rows, swizzled K-major
    static constexpr uint32_t kPhiBase = 0;
    static constexpr uint32_t kV1Base = kSlots * 2 * kPhiBytes;
    static constexpr uint32_t kOnes = kV1Base + kSlots * kVAtom;
    static constexpr uint32_t kKBase = kOnes + kVAtom;
    static constexpr uint32_t kBytes = kKBase + kKSlots * kK + 1024;
    static constexpr int kOutStride = kDV + 4;    // epilogue staging rows: 16-byte aligned, float4 conflict-free
    static_assert(kFT * kOutStride * 4 <= kV1Base, "epilogue staging fits the Phi_K slots");
};
constexpr int kStateThreads = kCompute + 32;

template <int D, int N>
__global__ void __launch_bounds__(kStateThreads, 2)
tcf_state_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                 float* __restrict__ W, int Ntok, int n, int F, int64_t stride, int G, int NG,
                 unsigned int* __restrict__ err) {
    using L = StSm<D>;
    constexpr int S4 = L::kSlots, KS = L::kKSlots;
    extern __shared__ uint8_t sm_raw[];
    uint8_t* sm = align1k(sm_raw);
    __shared__ __align__(8) uint64_t kload[KS], kfree[KS], vload[S4], full[S4], empty[S4];
    __shared__ uint32_t tslot;
    __shared__ int s_bad;
    volatile int* bad = &s_bad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, ft = blockIdx.y, bh = blockIdx.z;
    const int f0 = ft * kFT;
    const int nf = min(kFT, F - f0);
    const int64_t gt0 = (int64_t)g * G;
    const int gn = (int)min64(G, (int64_t)Ntok - gt0);
    const int nsub = (gn + kTok - 1) / kTok;
    auto phi = [&](int b) { return sm + L::kPhiBase + b * 2 * kPhiBytes; };
    auto v1s = [&](int b) { return sm + L::kV1Base + b * kVAtom; };
    auto krows = [&](int b) { return sm + L::kKBase + b * L::kK; };

    if (tid == 0) {
        for (int i = 0; i < KS; ++i) {
            ptx::mbar_init(&kload[i], 1);
            ptx::mbar_init(&kfree[i], kCompute / 2);
        }
        for (int i = 0; i < S4; ++i) {
            ptx::mbar_init(&vload[i], 1);
            ptx::mbar_init(&full[i], kCompute / 2);
            ptx::mbar_init(&empty[i], 1);
        }
        s_bad = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kCompute / 32) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    init_ones_atom(sm + L::kOnes, tid, kStateThreads);
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tacc = tslot;

    if (warp == kCompute / 32) {
        if (lane == 0) {
            // TMA producer and MMA issuer: issue whatever is ready, in order
            // within each kind (k loads, v loads, MMAs of a stage)
            int nk = 0, nv = 0, nm = 0;
            uint32_t idle = 0;
            while (nm < nsub) {
                bool prog = false;
                if (nk < nsub && (nk < KS || ptx::mbar_test(&kfree[nk % KS], ((nk / KS) - 1) & 1))) {
                    ptx::mbar_arrive_expect_tx(&kload[nk % KS], L::kK);
                    ptx::tma_load_3d(krows(nk % KS), &tmk, 0, (int)(gt0 + (int64_t)nk * kTok), bh, &kload[nk % KS]);
                    ++nk;
                    prog = true;
                }
                if (nv < nsub && (nv < S4 || ptx::mbar_test(&empty[nv % S4], ((nv / S4) - 1) & 1))) {
                    ptx::mbar_arrive_expect_tx(&vload[nv % S4], kVAtom);
                    ptx::tma_load_3d(v1s(nv % S4), &tmv, 0, (int)(gt0 + (int64_t)nv * kTok), bh, &vload[nv % S4]);
                    ++nv;
                    prog = true;
                }
                if (nm < nv && ptx::mbar_test(&full[nm % S4], (nm / S4) & 1) &&
                    ptx::mbar_test(&vload[nm % S4], (nm / S4) & 1)) {
                    fence_after_sync();
                    const uint8_t* ph = phi(nm % S4);
                    const uint32_t lbo = (uint32_t)(L::kOnes - (L::kV1Base + (nm % S4) * kVAtom));
                    const uint64_t ahd = smem_desc(ph, kLboFT, 128), ald = smem_desc(ph + kPhiBytes, kLboFT, 128);
                    const uint64_t bd = smem_desc_sw(v1s(nm % S4), lbo, 1024, kSwizzle128);
                    const uint32_t id = idesc_bf16(kFT, kNV, 1, 1);
                    // descriptors advance by constants: 2 K groups of Phi_K, 16 token rows of v
#pragma unroll
                    for (int ks = 0; ks < kTok / 16; ++ks) {
                        mma_bf16(tacc, ahd + (2 * kLboFT / 16) * ks, bd + 128 * ks, id, (nm > 0 || ks > 0) ? 1u : 0u);
                        mma_bf16(tacc, ald + (2 * kLboFT / 16) * ks, bd + 128 * ks, id, 1u);
                    }
                    mma_commit(&empty[nm % S4]);
                    ++nm;
                    prog = true;
                }
                if (prog) {
                    idle = 0;
                } else if (++idle > kWaitPolls || *bad) {
                    *bad = 1;
                    break;
                }
            }
            // the last commit covers every MMA issued; copies issued but never
            // consumed (only after a failure) must land before the CTA leaves
            if (nm > 0 && !ptx::mbar_wait(&empty[(nm - 1) % S4], ((nm - 1) / S4) & 1, kWaitPolls)) *bad = 1;
            for (int i = (nk > KS ? nk - KS : 0); i < nk; ++i)
                ptx::mbar_wait(&kload[i % KS], (i / KS) & 1, kWaitPolls);
            for (int i = (nv > S4 ? nv - S4 : 0); i < nv; ++i)
                ptx::mbar_wait(&vload[i % S4], (i / S4) & 1, kWaitPolls);
        }
    } else {
        // warpgroup w evaluates the features of stages w, w + 2, ...:
        // token t, features [64 h, 64 h + 64) of the tile
        const int w = warp >> 2, wt = tid & 127, t = wt & (kTok - 1), h = wt >> 6;
        for (int s = w; s < nsub; s += 2) {
            const int kb = s % KS, b = s % S4;
            if (!waitb(&kload[kb], (s / KS) & 1, bad)) break;
            float o[64];
            const uint8_t* rowbase = krows(kb) + t * RowSw<D>::kRowBytes;
            const uint32_t sw = swizzle_of_row(t, RowSw<D>::kRowBytes);
            fe::Eval<D, N, false>::block(ft * 4 + h * 2, rowbase, sw, nullptr, n, F, 0.f,
                                         *reinterpret_cast<float(*)[32]>(o));
            fe::Eval<D, N, false>::block(ft * 4 + h * 2 + 1, rowbase, sw, nullptr, n, F, 0.f,
                                         *reinterpret_cast<float(*)[32]>(o + 32));
            ptx::mbar_arrive(&kfree[kb]);
            if (t >= min(kTok, gn - s * kTok)) {  // zero-filled rows past the sequence: phi(0) has a constant feature
#pragma unroll
                for (int e = 0; e < 64; ++e) o[e] = 0.f;
            }
            if (s >= S4 && !waitb(&empty[b], ((s / S4) - 1) & 1, bad)) break;
            uint8_t* ph = phi(b);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t off = mnmaj(t, h * 8 + i, kLboFT);
                store_split8(o + 8 * i, ph + off, ph + kPhiBytes + off);
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(&full[b]);
        }
    }
    __syncthreads();
    fence_after_sync();
    const bool ok = s_bad == 0;

    // TMEM lane j holds feature f0 + j: columns 0..63 its S_v row, 64 its z
    float* Wg = W + ((int64_t)bh * NG + g) * stride;
    float* sOut = reinterpret_cast<float*>(sm);
    if (ok && tid < kCompute) {
        const int row = (warp & 3) * 32 + lane, half = warp >> 2;
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
    }
    if (!ok && tid == 0) atomicOr(err, kErrPrefillPipe);
    fence_before_sync();
    __syncthreads();
    if (ok) {
        float4* dst = reinterpret_cast<float4*>(Wg + (int64_t)f0 * kDV);
        for (int e = tid; e < nf * (kDV / 4); e += kStateThreads) {
            const int j = e / (kDV / 4), c = e % (kDV / 4);
            dst[e] = *reinterpret_cast<const float4*>(sOut + j * L::kOutStride + c * 4);
        }
    }
    if (warp == kCompute / 32) {
        fence_after_sync();
        tmem_dealloc(tacc, 128);
    }
}

// ---------------------------------------------------------------- 2 + 3. scan and operand tiles in one pass
// The exclusive scan over the NG group states of a head fused with their
// packing into read-out operand tiles: S_<g (fp32, the library's state
// layout) becomes, for each 64-feature tile r, one MN-major bf16 operand
// [K = 64 features][N = 160] (columns 0..79 the hi parts, 80..159 the lo
// parts, of [S_v row | z | 0 ...]; features past F zero).  A thread owns 8 columns of one feature
// row (its 16-byte unit of a tile row, hi and lo) and walks the groups,
// writing the prefix before group g as group g's tile unit, then adding group
// g's state.  The group states are read once and the exclusive prefixes never
// go back to memory; the total goes to state_out (padding zero-filled by the
// head's first block).  Units are ordered so that 8 consecutive threads fill
// one 128-byte line of a tile (8 feature rows of one column group).
__global__ void __launch_bounds__(256)
tcf_scan_pack_kernel(const float* __restrict__ W, const float* __restrict__ state_in, float* __restrict__ state_out,
                     uint8_t* __restrict__ PK, int F, int64_t stride, int NG, int R, int g0) {
    ptx::pdl_wait_primary();
    ptx::pdl_launch_dependents();
    const int bh = blockIdx.y;
    const int u = blockIdx.x * 256 + threadIdx.x;
    const int f8 = u / 80, rem = u % 80, gq = rem >> 3, f = f8 * 8 + (rem & 7);
    if (f < R * kRT) {
        const int r = f / kRT, j = f % kRT;
        const bool live = f < F && gq < 9;
        const float* Sb = W + (int64_t)bh * NG * stride;
        float run[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        auto ld8 = [&](const float* S, float (&x)[8]) {
            if (gq < 8) {
                const float4 a = __ldg(reinterpret_cast<const float4*>(S + (int64_t)f * kDV + gq * 8));
                const float4 b = __ldg(reinterpret_cast<const float4*>(S + (int64_t)f * kDV + gq * 8) + 1);
                x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
                x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
            } else {
                x[0] = __ldg(S + (int64_t)F * kDV + f);
#pragma unroll
                for (int i = 1; i < 8; ++i) x[i] = 0.f;
            }
        };
        if (live && state_in) ld8(state_in + (int64_t)bh * stride, run);
        for (int g = 0; g < NG; ++g) {
            if (g >= g0) {
                uint8_t* dst = PK + (((int64_t)bh * NG + g) * R + r) * kSTile;
                store_split8(run, dst + mnmaj(j, gq, kLboS), dst + mnmaj(j, 10 + gq, kLboS));
            }
            if (live) {
                float x[8];
                ld8(Sb + (int64_t)g * stride, x);
#pragma unroll
                for (int i = 0; i < 8; ++i) run[i] += x[i];
            }
        }
        if (live && state_out) {
            float* so = state_out + (int64_t)bh * stride;
            if (gq < 8) {
                reinterpret_cast<float4*>(so + (int64_t)f * kDV + gq * 8)[0] = make_float4(run[0], run[1], run[2], run[3]);
                reinterpret_cast<float4*>(so + (int64_t)f * kDV + gq * 8)[1] = make_float4(run[4], run[5], run[6], run[7]);
            } else {
                so[(int64_t)F * kDV + f] = run[0];
            }
        }
    }
    if (state_out && blockIdx.x == 0)
        for (int64_t e = (int64_t)F * (kDV + 1) + threadIdx.x; e < stride; e += 256)
            state_out[(int64_t)bh * stride + e] = 0.f;
}

// ---------------------------------------------------------------- 4. outputs
template <int D>
struct OutSm {
    static constexpr uint32_t kQop = kQ * D * 2;  // Q, swizzled K-major
    static constexpr uint32_t kKt = kTok * D * 2; // key tile, swizzled K-major
    static constexpr uint32_t kKV = kKt + kVAtom;
    static constexpr int kKVSlots = 4, kSSlots = 4;
    static constexpr uint32_t kKVbase = kQop;
    static constexpr uint32_t kOnes = kKVbase + kKVSlots * kKV;
    static constexpr uint32_t kSbase = kOnes + kVAtom;
    static constexpr uint32_t kBytes = kSbase + kSSlots * kSTile + 1024;
};
// two warpgroups of eight warps (two per TMEM lane quadrant, each taking half
// of a tile's columns), then the hi-operand PV/read-out MMA warp, the q/k/v
// and S producer warps, and the warp that issues the scores MMAs and the
// lo-operand PV/read-out MMAs
constexpr int kOutCompute = 512;
constexpr int kOutThreads = kOutCompute + 128;
constexpr int kWMma = kOutCompute / 32, kWLoad = kWMma + 1, kWSLoad = kWMma + 2, kWMma2 = kWMma + 3;

template <int D, int N>
__global__ void __launch_bounds__(kOutThreads, 1)
tcf_out_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, const uint8_t* __restrict__ PK, float* __restrict__ out,
               int Ntok, int n, float tau, int F, int G, int NG, int R, int carried,
               unsigned int* __restrict__ err) {
    using L = OutSm<D>;
    extern __shared__ uint8_t sm_raw[];
    uint8_t* sm = align1k(sm_raw);
    __shared__ __align__(8) uint64_t q_loaded, kv_loaded[L::kKVSlots], kv_empty[L::kKVSlots], sc_full[2], sc_free[2],
        pp_full[2], pp_free[2], s_loaded[L::kSSlots], s_empty[L::kSSlots], o_done[2];
    __shared__ uint32_t tslot;
    __shared__ int s_bad;
    volatile int* bad = &s_bad;
    uint8_t* sQ = sm;
    auto kv = [&](int slot) { return sm + L::kKVbase + slot * L::kKV; };
    auto sS = [&](int slot) { return sm + L::kSbase + slot * kSTile; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, bh = blockIdx.y;
    const int64_t q0 = (int64_t)qt * kQ;
    const int nq = (int)min64(kQ, (int64_t)Ntok - q0);
    const int g = (int)(q0 / G);
    const int64_t gs = (int64_t)g * G;
    const int64_t kend = min64(q0 + kQ, (int64_t)Ntok);
    const int T = (int)((kend - gs + kTok - 1) / kTok);  // key tiles, >= 1
    const int Rr = (g > 0 || carried) ? R : 0;           // read-out tiles
    TA_PHASE_VARS(ph_start);
    TA_PHASE_T0(ph_start);

    if (tid == 0) {
        ptx::mbar_init(&q_loaded, 1);
        for (int i = 0; i < L::kKVSlots; ++i) {
            ptx::mbar_init(&kv_loaded[i], 1);
            ptx::mbar_init(&kv_empty[i], 2);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&sc_full[i], 1);
            ptx::mbar_init(&sc_free[i], kOutCompute / 2);
            ptx::mbar_init(&pp_full[i], kOutCompute / 2);
            ptx::mbar_init(&pp_free[i], 2);
        }
        for (int i = 0; i < L::kSSlots; ++i) {
            ptx::mbar_init(&s_loaded[i], 1);
            ptx::mbar_init(&s_empty[i], 2);
        }
        ptx::mbar_init(&o_done[0], 1);
        ptx::mbar_init(&o_done[1], 1);
        s_bad = 0;
        ptx::fence_mbar_init();
    }
    if (warp == kWMma) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    init_ones_atom(sm + L::kOnes, tid, kOutThreads);
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    // TMEM (all 512 columns): scores of two key tiles (0..127); O_hi in
    // 128..287, whose columns 0..79 take P_hi [V|1] + Phi_Q,hi S_hi and 80..159
    // Phi_Q,hi S_lo; O_lo in 288..367 takes P_lo [V|1] + Phi_Q,lo S_hi; per
    // warpgroup one A operand (P or Phi_Q, hi in 32 columns then lo in 32) at
    // 384 + 64 w.  O = O_hi[0:80] + O_hi[80:160] + O_lo.
    const uint32_t tS = tslot, tO = tslot + 128, tO2 = tslot + 288;
    auto tA = [&](int w) { return tslot + 384u + 64u * (uint32_t)w; };

    if (warp == kWLoad) {
        if (lane == 0) {
            // q once, then key/value tiles through a ring of three slots
            ptx::mbar_arrive_expect_tx(&q_loaded, L::kQop);
            ptx::tma_load_3d(sQ, &tmq, 0, (int)q0, bh, &q_loaded);
            int ld = 0;
            for (; ld < T; ++ld) {
                const int slot = ld % L::kKVSlots;
                if (ld >= L::kKVSlots && !waitb(&kv_empty[slot], ((ld / L::kKVSlots) - 1) & 1, bad)) break;
                uint8_t* st = kv(slot);
                ptx::mbar_arrive_expect_tx(&kv_loaded[slot], L::kKV);
                const int y = (int)(gs + (int64_t)ld * kTok);
                ptx::tma_load_3d(st, &tmk, 0, y, bh, &kv_loaded[slot]);
                ptx::tma_load_3d(st + L::kKt, &tmv, 0, y, bh, &kv_loaded[slot]);
            }
            // every issued copy lands before the CTA can leave
            ptx::mbar_wait(&q_loaded, 0, kWaitPolls);
            for (int li = (ld > L::kKVSlots ? ld - L::kKVSlots : 0); li < ld; ++li)
                ptx::mbar_wait(&kv_loaded[li % L::kKVSlots], (li / L::kKVSlots) & 1, kWaitPolls);
        }
    } else if (warp == kWSLoad) {
        // waits for the preceding kernels even without a read-out, so that
        // this grid completes only after they have
        if (lane == 0) ptx::pdl_wait_primary();
        if (lane == 0 && Rr > 0) {
            const uint8_t* src = PK + ((int64_t)bh * NG + g) * R * kSTile;
            int ld = 0;
            for (; ld < Rr; ++ld) {
                const int slot = ld % L::kSSlots;
                if (ld >= L::kSSlots && !waitb(&s_empty[slot], ((ld / L::kSSlots) - 1) & 1, bad)) break;
                ptx::mbar_arrive_expect_tx(&s_loaded[slot], kSTile);
                ptx::bulk_g2s(sS(slot), src + (int64_t)ld * kSTile, kSTile, &s_loaded[slot]);
            }
            for (int li = (ld > L::kSSlots ? ld - L::kSSlots : 0); li < ld; ++li)
                ptx::mbar_wait(&s_loaded[li % L::kSSlots], (li / L::kSSlots) & 1, kWaitPolls);
        }
    } else if (warp == kWMma || warp == kWMma2) {
        if (lane == 0) {
            // PV and read-out MMAs, in order: role 0 multiplies the hi halves
            // of P / Phi_Q into O_hi, role 1 the lo halves into O_lo
            const int role = warp == kWMma ? 0 : 1;
            const uint32_t dst = role == 0 ? tO : tO2;
            TA_PHASE_VARS(m_t, m_ppfull = 0, m_sl = 0, m_issue = 0);
            const uint32_t id80 = idesc_bf16(kQ, kNV, 0, 1);
            const uint32_t idro = idesc_bf16(kQ, role == 0 ? 2 * kNV : kNV, 0, 1);
            // role 1 also issues the scores S_t = Q K_t^T into TMEM buffer t & 1
            using RS = RowSw<D>;
            const uint64_t qd = smem_desc_sw(sQ, 16, RS::kSbo, RS::kLayout);
            const uint32_t ids = idesc_bf16(kQ, kTok, 0, 0);
            auto scores = [&](int t) -> bool {
                const int slot = t % L::kKVSlots;
                if (!waitb(&kv_loaded[slot], (t / L::kKVSlots) & 1, bad)) return false;
                fence_after_sync();
                const uint64_t kd = smem_desc_sw(kv(slot), 16, RS::kSbo, RS::kLayout);
                const uint32_t d = tS + (uint32_t)((t & 1) * kTok);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) mma_bf16(d, qd + 2 * ks, kd + 2 * ks, ids, ks > 0 ? 1u : 0u);
                mma_commit(&sc_full[t & 1]);
                return true;
            };
            bool go = true;
            if (role == 1) {
                go = waitb(&q_loaded, 0, bad);
                if (go) go = scores(0);
                if (go && T > 1) go = scores(1);
            }
            for (int t = 0; t < T && go; ++t) {
                const int w = t & 1, slot = t % L::kKVSlots;
                // scores of tile t + 2 go ahead of PV(t) once the warpgroup has
                // read the scores of tile t, if the key tile is already resident
                bool early = false;
                if (role == 1 && t + 2 < T) {
                    if (!waitb(&sc_free[w], (t >> 1) & 1, bad)) {
                        go = false;
                        break;
                    }
                    if (ptx::mbar_test(&kv_loaded[(t + 2) % L::kKVSlots], ((t + 2) / L::kKVSlots) & 1)) {
                        if (!scores(t + 2)) {
                            go = false;
                            break;
                        }
                        early = true;
                    }
                }
                TA_PHASE_T0(m_t);
                if (!waitb(&pp_full[w], (t >> 1) & 1, bad)) {
                    go = false;
                    break;
                }
                TA_PHASE_ACC(m_ppfull, m_t);
                TA_PHASE_T0(m_t);
                fence_after_sync();
                const uint32_t a = tA(w) + 32u * role;
                const uint32_t lbo = (uint32_t)(L::kOnes - (L::kKVbase + slot * L::kKV + L::kKt));
                const uint64_t vd = smem_desc_sw(kv(slot) + L::kKt, lbo, 1024, kSwizzle128);
#pragma unroll
                for (int ks = 0; ks < kTok / 16; ++ks)
                    mma_bf16_ts(dst, a + ks * 8, vd + 128 * ks, id80, (t > 0 || ks > 0) ? 1u : 0u);
                mma_commit(&pp_free[w]);
                mma_commit(&kv_empty[slot]);  // scores(t) completed before P(t) existed
                TA_PHASE_ACC(m_issue, m_t);
                if (role == 1 && t + 2 < T && !early && !scores(t + 2)) go = false;
            }
            const int nuse[2] = {(T + 1) / 2, T / 2};
            for (int r = 0; r < Rr && go; ++r) {
                const int w = r & 1, u = nuse[w] + (r >> 1), slot = r % L::kSSlots;
                TA_PHASE_T0(m_t);
                if (!waitb(&pp_full[w], u & 1, bad)) {
                    go = false;
                    break;
                }
                TA_PHASE_ACC(m_ppfull, m_t);
                TA_PHASE_T0(m_t);
                if (!waitb(&s_loaded[slot], (r / L::kSSlots) & 1, bad)) {
                    go = false;
                    break;
                }
                TA_PHASE_ACC(m_sl, m_t);
                TA_PHASE_T0(m_t);
                fence_after_sync();
                const uint32_t a = tA(w) + 32u * role;
                const uint64_t sd = smem_desc(sS(slot), kLboS, 128);
#pragma unroll
                for (int ks = 0; ks < kRT / 16; ++ks) mma_bf16_ts(dst, a + ks * 8, sd + (2 * kLboS / 16) * ks, idro, 1u);
                mma_commit(&pp_free[w]);
                mma_commit(&s_empty[slot]);
                TA_PHASE_ACC(m_issue, m_t);
            }
            mma_commit(&o_done[role]);  // covers every MMA this thread issued
            if (!ptx::mbar_wait(&o_done[role], 0, kWaitPolls)) *bad = 1;
            TA_PHASE_PUT(0, 1, role == 0, m_ppfull);
            TA_PHASE_PUT(0, 4, role == 0, m_sl);
            TA_PHASE_PUT(0, 5, role == 0, m_issue);
        }
    } else {
        // warpgroup w: P of key tiles w, w + 2, ..., then Phi_Q of read-out
        // tiles w, w + 2, ...; thread = query row, half hh of the tile's 64
        // columns (keys or features)
        const int w = warp >> 3, hh = (warp >> 2) & 1;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const int64_t qi = q0 + row;
        float qc[kMaxN];
#pragma unroll
        for (int m = 0; m < kMaxN; ++m) qc[m] = query_coeff(m, tau);
        const uint32_t a_hi = tA(w) + lane_off + 16 * hh, a_lo = a_hi + 32;
        if (w == 0 && hh == 0) {  // O columns 80..159 start at zero (the MMAs into them accumulate)
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0;
            tmem_st32(tO + lane_off + 80, z);
            tmem_st32(tO + lane_off + 112, z);
            tmem_st16(tO + lane_off + 144, *reinterpret_cast<uint32_t(*)[16]>(z));
            tmem_st_wait();
            fence_before_sync();
        }
        int u = 0;
        TA_PHASE_VARS(w_t, w_sc = 0, w_p = 0, w_pf = 0, w_st = 0, w_phi = 0, w_pf2 = 0);
        for (int t = w; t < T; t += 2, ++u) {
            TA_PHASE_T0(w_t);
            if (!waitb(&sc_full[w], (t >> 1) & 1, bad)) break;
            TA_PHASE_ACC(w_sc, w_t);
            TA_PHASE_T0(w_t);
            fence_after_sync();
            float s[32];
            tmem_ld32(tS + lane_off + w * kTok + 32 * hh, s);
            tmem_ld_wait();
            fence_before_sync();
            ptx::mbar_arrive(&sc_free[w]);
            const int64_t k0 = gs + (int64_t)t * kTok + 32 * hh;
            const bool mask = k0 + 31 > q0 || k0 + 32 > Ntok;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float x = s[j];
                float p;
                if constexpr (N > 0) {
                    p = qc[N - 1];
#pragma unroll
                    for (int m = N - 2; m >= 0; --m) p = fmaf(p, x, qc[m]);
                } else {
                    p = qc[n - 1];
                    for (int m = n - 2; m >= 0; --m) p = fmaf(p, x, qc[m]);
                }
                if (mask && !(k0 + j <= qi && k0 + j < kend)) p = 0.f;
                s[j] = p;
            }
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) split2(s[2 * i], s[2 * i + 1], hi[i], lo[i]);
            TA_PHASE_ACC(w_p, w_t);
            TA_PHASE_T0(w_t);
            if (u > 0 && !waitb(&pp_free[w], (u - 1) & 1, bad)) break;
            TA_PHASE_ACC(w_pf, w_t);
            TA_PHASE_T0(w_t);
            fence_after_sync();
            tmem_st16(a_hi, hi);
            tmem_st16(a_lo, lo);
            tmem_st_wait();
            fence_before_sync();
            ptx::mbar_arrive(&pp_full[w]);
            TA_PHASE_ACC(w_st, w_t);
        }
        // q must be resident before Phi_Q is read from it: a warpgroup
        // without key tiles (T == 1) reaches this point before any scores
        // MMA, hence before anything else has waited for the q load
        if (Rr > 0 && !waitb(&q_loaded, 0, bad)) *bad = 1;
        if (!*bad) {
            const uint8_t* rowbase = sQ + row * RowSw<D>::kRowBytes;
            const uint32_t sw = swizzle_of_row(row, RowSw<D>::kRowBytes);
            for (int r = w; r < Rr; r += 2, ++u) {
                float o[32];
                TA_PHASE_T0(w_t);
                fe::Eval<D, N, true>::block(r * 2 + hh, rowbase, sw, qc, n, F, tau, o);
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) split2(o[2 * i], o[2 * i + 1], hi[i], lo[i]);
                TA_PHASE_ACC(w_phi, w_t);
                TA_PHASE_T0(w_t);
                if (u > 0 && !waitb(&pp_free[w], (u - 1) & 1, bad)) break;
                TA_PHASE_ACC(w_pf2, w_t);
                TA_PHASE_T0(w_t);
                fence_after_sync();
                tmem_st16(a_hi, hi);
                tmem_st16(a_lo, lo);
                tmem_st_wait();
                fence_before_sync();
                ptx::mbar_arrive(&pp_full[w]);
                TA_PHASE_ACC(w_st, w_t);
            }
        }
        TA_PHASE_PUT(0, 6, tid == 0, w_sc);
        TA_PHASE_PUT(0, 7, tid == 0, w_p);
        TA_PHASE_PUT(0, 8, tid == 0, w_pf);
        TA_PHASE_PUT(0, 9, tid == 0, w_st);
        TA_PHASE_PUT(0, 10, tid == 0, w_phi);
        TA_PHASE_PUT(0, 11, tid == 0, w_pf2);
    }
    __syncthreads();  // the MMA thread has seen every MMA complete (or a failure)
    TA_PHASE_PUT(0, 12, tid == 0, (unsigned long long)T);
    TA_PHASE_PUT(0, 13, tid == 0, (unsigned long long)Rr);
    TA_PHASE_VARS(ph_end);
    TA_PHASE_T0(ph_end);
    TA_PHASE_PUT(0, 0, tid == 0, ph_end - ph_start);
    fence_after_sync();
    const bool ok = s_bad == 0;
    if (ok && tid < kOutCompute) {
        // warp (quadrant q, column block cb): rows 32 q .., output columns 16 cb ..
        const int row = (warp & 3) * 32 + lane, cb = warp >> 2;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        float o[16], o2[16];
        tmem_ld16(tO + lane_off + 16 * cb, o);
        tmem_ld16(tO + lane_off + kNV + 16 * cb, o2);
        const float d1 = tmem_ld1(tO + lane_off + kDV), d2 = tmem_ld1(tO + lane_off + kNV + kDV);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] += o2[i];
        tmem_ld16(tO2 + lane_off + 16 * cb, o2);
        const float d3 = tmem_ld1(tO2 + lane_off + kDV);
        tmem_ld_wait();
        if (row < nq) {
            const float rcp = __frcp_rn(d1 + d2 + d3);
            float4* dst = reinterpret_cast<float4*>(out + ((int64_t)bh * Ntok + q0 + row) * kDV + 16 * cb);
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = (o[i] + o2[i]) * rcp;
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
        }
    }
    if (!ok && tid == 0) atomicOr(err, kErrPrefillPipe);
    fence_before_sync();
    __syncthreads();
    if (warp == kWMma) {
        fence_after_sync();
        tmem_dealloc(tslot, 512);
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
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StSm<D>::kBytes);
        // two CTAs an SM (each allocates 128 TMEM columns): the largest shared-memory carveout
        if (res[dev] == cudaSuccess)
            res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_state_kernel<D, N>),
                                            cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (res[dev] == cudaSuccess)
            res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_out_kernel<D, N>),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OutSm<D>::kBytes);
    });
    if (res[dev] != cudaSuccess) return TAYLOR_ERR_CUDA;

    CUtensorMap tmq, tmk, tmv;
    if (make_tmap_bf16_3d(&tmq, q, D, (uint64_t)Ntok, (uint64_t)BH, D, kQ, D * 2) != cudaSuccess ||
        make_tmap_bf16_3d(&tmk, k, D, (uint64_t)Ntok, (uint64_t)BH, D, kTok, D * 2) != cudaSuccess ||
        make_tmap_bf16_3d(&tmv, v, kDV, (uint64_t)Ntok, (uint64_t)BH, kDV, kTok, 128) != cudaSuccess)
        return kNotApplicable;

    // group size: about F tokens (the pairwise work of a query tile then
    // stays below its read-out work), in [128, 2048], no larger than needed
    int G = 128;
    while (G < 2048 && 2 * (int64_t)G <= F) G *= 2;
    while (G > 128 && G / 2 >= Ntok) G /= 2;
    const int NG = (Ntok + G - 1) / G;
    const int NFT = (int)((F + kFT - 1) / kFT);
    const int R = (int)((F + kRT - 1) / kRT);
    const bool need_ws = NG > 1 || state_in || state_out;
    const int g0 = state_in ? 0 : 1;  // first group whose outputs read a state
    const bool need_pk = NG > g0;
    const size_t w_bytes = ((size_t)BH * NG * stride * sizeof(float) + 1023) / 1024 * 1024;
    const size_t pk_bytes = need_pk ? (size_t)BH * NG * R * kSTile : 0;
    uint8_t* ws = nullptr;
    if (need_ws) {
        if (workspace_alloc(reinterpret_cast<void**>(&ws), w_bytes + pk_bytes, stream) != cudaSuccess) {
            cudaGetLastError();
            return TAYLOR_ERR_OUT_OF_MEMORY;
        }
    }
    float* Wb = reinterpret_cast<float*>(ws);
    uint8_t* PKb = need_pk ? ws + w_bytes : nullptr;
    cudaError_t e = cudaSuccess;
    if (need_ws) {
        TA_TIMED(stream, "tcf_state_kernel",
                 tcf_state_kernel<D, N><<<dim3(NG, NFT, BH), kStateThreads, StSm<D>::kBytes, stream>>>(
                     tmk, tmv, Wb, Ntok, n, (int)F, stride, G, NG, err));
        e = cudaGetLastError();
        // the scan and the operand tiles in one pass: 8 columns of a feature
        // row a thread, 10 column groups a row (hi 0..7, z, zero), rows to 64 R
        if (e == cudaSuccess) {
            const int units = R * kRT * 10;
            TA_TIMED(stream, "tcf_scan_pack_kernel",
                     e = launch_maybe_pdl(tcf_scan_pack_kernel, dim3((units + 255) / 256, BH), dim3(256), 0, stream,
                                          true, (const float*)Wb, state_in, state_out, PKb, (int)F, stride, NG, R,
                                          need_pk ? g0 : NG));
        }
    }
    if (e == cudaSuccess) {
        const int NQ = (Ntok + kQ - 1) / kQ;
        TA_TIMED(stream, "tcf_out_kernel",
                 e = launch_maybe_pdl(tcf_out_kernel<D, N>, dim3(NQ, BH), dim3(kOutThreads), OutSm<D>::kBytes, stream,
                                      need_ws, tmq, tmk, tmv, (const uint8_t*)PKb, out, Ntok, n, tau, (int)F, G, NG, R,
                                      state_in != nullptr ? 1 : 0, err));
        if (e == cudaSuccess) e = cudaGetLastError();
    }
    if (ws) {
        const cudaError_t e2 = workspace_free(ws, stream);
        if (e == cudaSuccess) e = e2;
    }
    if (e == cudaSuccess) return TAYLOR_OK;
    return e == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
}

}  // namespace tcf
}  // namespace tc
}  // namespace ta
