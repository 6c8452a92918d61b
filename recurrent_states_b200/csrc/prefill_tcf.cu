// Chunked causal prefill on the sm_100a tensor cores for any number of
// features: d_k in {16, 32, 64}, 1 <= n <= 5, d_v = 64, bf16 inputs.  The
// state does not fit one SM at these widths (2,145 features at d_k 64, n 3;
// 4,845 at d_k 16, n 5), so the feature dimension is cut into tiles of 128.
//
// Method (arXiv 2610.20637, abstract): the state S = sum_j phi(k_j)[v_j|1]^T
// is additive across chunks, so prefill is a scan over group states.
// Tokens are cut into groups of G (a multiple of 128); then
//   1. tcf_state_kernel (group, feature tile, head):
//        dS_g[tile, :] = Phi_K[:, tile]^T (128 x G) . [V|1|0] (G x 80),
//        accumulated over the group's 128-token sub-chunks in TMEM;
//   2. the scan over groups (shared with the other paths);
//   3. tcf_out_kernel (128 query tokens, head):
//        O = sum over key tiles of the group up to the diagonal of
//              (poly(tau Q K^T) (.) mask) [V|1|0]
//          + sum over feature tiles of (c (.) Phi_Q[:, tile]) S_<g[tile, :],
//        o = O[:, :64] * (1 / O[:, 64]).
// Every contraction is a tcgen05.mma chain (bf16 operands in shared memory,
// fp32 accumulators in TMEM); operands produced in fp32 (Phi_K, Phi_Q, P and
// S_<g) are split into hi/lo bf16 pairs as in the d_k 16 kernels, so about 16
// significant bits reach the fp32 accumulators.  Each step stages its
// operands, one thread issues the MMAs and commits them to an mbarrier that
// the block waits on (bounded) before the next step reuses shared memory.
#include <mutex>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "feature_table.cuh"
#include "internal.h"
#include "prefill_tc.h"
#include "ptx.cuh"
#include "tcgen05.cuh"

namespace ta {
namespace tc {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kC = 128;        // tokens per tile (MMA M, or K of the state update)
constexpr int kFT = 128;       // features per tile
constexpr int kDV = 64;
constexpr int kNV = 80;        // [V | 1 | 0 ...]
constexpr int kThreads = 256;
constexpr uint32_t kWaitPolls = 1u << 24;

constexpr uint32_t kLbo128 = 16 * 128;        // K-group stride of an MN-major operand 128 wide
constexpr uint32_t kLboNV = (kNV / 8) * 128;  // K-group stride of an MN-major operand 80 wide
constexpr uint32_t kSbo128 = 16 * 128;        // row-group stride of a K-major operand 128 deep

// token vectors in fp32, rows padded to an odd stride so that 32 threads on
// 32 tokens reading the same coordinate hit 32 banks
template <int D>
struct XS {
    static constexpr int kStride = D + 1;
    static constexpr uint32_t kBytes = (uint32_t)(kC * kStride * 4 + 127) / 128 * 128;
};

__device__ __forceinline__ float eval_tile(const FeatDesc& fd, const float* x) {
    if (fd.m < 0) return 0.f;
    return eval_desc(fd, x);
}

// Descriptors of features [f0, f0 + 128) of (d, n), zero features past F.
__device__ __forceinline__ void load_tile_desc(FeatDesc* ds, int d, int n, int f0, int F, float tau,
                                               const float* qc, bool query) {
    const int j = threadIdx.x;
    if (j < kFT) {
        if (f0 + j < F) {
            ds[j] = get_desc(feat_table(d, n), d, n, f0 + j, tau, qc, query);
        } else {
            FeatDesc z;
            z.m = -1;
            z.packed = 0;
            z.w = 0.f;
            ds[j] = z;
        }
    }
}

// Rows of a [*, D] bf16 tensor -> fp32 X rows (t < valid, else zeros).
template <int D>
__device__ __forceinline__ void stage_x(float* xs, const bf16* src, int valid) {
    for (int e = threadIdx.x; e < kC * D; e += kThreads) {
        const int t = e / D, i = e % D;
        xs[t * XS<D>::kStride + i] = t < valid ? __bfloat162float(src[(int64_t)t * D + i]) : 0.f;
    }
}

// A K-major bf16 operand [128 rows][D] from token rows (zeros past `valid`).
template <int D>
__device__ __forceinline__ void stage_kmajor_rows(uint8_t* dst, const bf16* src, int valid) {
    constexpr int G8 = D / 8;
    for (int e = threadIdx.x; e < kC * G8; e += kThreads) {
        const int t = e / G8, g = e % G8;
        const uint4 val = t < valid ? __ldg(reinterpret_cast<const uint4*>(src + (int64_t)t * D) + g)
                                    : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(dst + kmaj(t, g, (uint32_t)G8 * 128u)) = val;
    }
}

// [v | 1 | 0...] rows for 128 tokens as an MN-major operand whose K is the
// token and whose MN is the column; `groups` 8-column groups wide (10 for
// the N = 80 B operand, 16 for the M = 128 A operand of the state update).
__device__ __forceinline__ void stage_v1(uint8_t* dst, const bf16* v, int valid, int groups, uint32_t lbo) {
    for (int e = threadIdx.x; e < kC * groups; e += kThreads) {
        const int t = e / groups, g = e % groups;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (t < valid) {
            if (g < 8) val = __ldg(reinterpret_cast<const uint4*>(v + (int64_t)t * kDV) + g);
            else if (g == 8) val = make_uint4(0x3F80u, 0, 0, 0);  // bf16 1.0 in column 64
        }
        *reinterpret_cast<uint4*>(dst + mnmaj(t, g, lbo)) = val;
    }
}

__device__ __forceinline__ bool wait_block(uint64_t* bar, uint32_t parity) {
    const bool ok = ptx::mbar_wait(bar, parity, kWaitPolls);
    return __syncthreads_and(ok) != 0;
}

__device__ __forceinline__ void publish_smem() {
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
}

// ---------------------------------------------------------------- 1. group states
// dS_g[tile, :] = Phi_K[:, tile]^T (128 features x G tokens) . [V|1|0] (G x 80):
// M = 128 features (A MN-major, K = token), N = 80, accumulated in TMEM.
template <int D>
struct StateSmem {
    static constexpr uint32_t kX = 0;
    static constexpr uint32_t kV1 = kX + XS<D>::kBytes;            // [V|1|0], MN-major K=128 x 80
    static constexpr uint32_t kAh = kV1 + kC * kNV * 2;             // Phi_K tile, MN-major K=128 x 128
    static constexpr uint32_t kAl = kAh + kC * kFT * 2;
    static constexpr uint32_t kDesc = kAl + kC * kFT * 2;
    static constexpr uint32_t kBytes = kDesc + kFT * (uint32_t)sizeof(FeatDesc);
    static constexpr int kOutStride = kDV + 4;                      // staging rows: 16-byte aligned, float4 conflict-free
    static_assert(kFT * kOutStride * 4 <= 2 * kC * kFT * 2, "staging fits the Phi_K buffers");
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tcf_state_kernel(const bf16* __restrict__ k, const bf16* __restrict__ v, float* __restrict__ W, int N, int n,
                 int F, int64_t stride, int G, int NG, unsigned int* __restrict__ err) {
    using L = StateSmem<D>;
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb;
    __shared__ uint32_t tslot;
    float* xs = reinterpret_cast<float*>(sm + L::kX);
    uint8_t* sV1 = sm + L::kV1;
    uint8_t* sAh = sm + L::kAh;
    uint8_t* sAl = sm + L::kAl;
    FeatDesc* ds = reinterpret_cast<FeatDesc*>(sm + L::kDesc);
    float* sOut = reinterpret_cast<float*>(sm + L::kAh);  // reused after the last MMA

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = blockIdx.x, ft = blockIdx.y, bh = blockIdx.z;
    const int f0 = ft * kFT;
    const int nf = min(kFT, F - f0);
    const int64_t gt0 = (int64_t)g * G;
    const int gn = (int)min64(G, (int64_t)N - gt0);  // tokens in this group
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;

    if (tid == 0) {
        ptx::mbar_init(&mb, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tslot, 128);
        tmem_relinquish();
    }
    load_tile_desc(ds, D, n, f0, F, 0.f, nullptr, false);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tbase = tslot;

    bool ok = true;
    uint32_t parity = 0;
    const int nsub = (gn + kC - 1) / kC;
    for (int s = 0; s < nsub; ++s) {
        const int64_t t0 = gt0 + (int64_t)s * kC;
        const int valid = (int)min64(kC, (int64_t)N - t0);
        const bf16* kb = k + ((int64_t)bh * N + t0) * D;
        const bf16* vb = v + ((int64_t)bh * N + t0) * kDV;
        stage_x<D>(xs, kb, valid);
        stage_v1(sV1, vb, valid, 10, kLboNV);
        __syncthreads();
        // token `row`, features half*64 .. +64: one K row of the MN-major A operand
        // (padding tokens get phi(0); their [v|1] row is zero)
        {
            const float* x = xs + row * XS<D>::kStride;
#pragma unroll
            for (int g8 = 0; g8 < 8; ++g8) {
                const int j0 = half * 64 + g8 * 8;
                float buf[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) buf[e] = eval_tile(ds[j0 + e], x);
                uint4 hi, lo;
                split8(buf, hi, lo);
                *reinterpret_cast<uint4*>(sAh + mnmaj(row, j0 / 8, kLbo128)) = hi;
                *reinterpret_cast<uint4*>(sAl + mnmaj(row, j0 / 8, kLbo128)) = lo;
            }
        }
        publish_smem();
        if (tid == 0) {
            const uint32_t id = idesc_bf16(kFT, kNV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks) {
                const uint64_t b = smem_desc(sV1 + ks * 2 * kLboNV, kLboNV, 128);
                mma_bf16(tbase, smem_desc(sAh + ks * 2 * kLbo128, kLbo128, 128), b, id, (s > 0 || ks > 0) ? 1u : 0u);
                mma_bf16(tbase, smem_desc(sAl + ks * 2 * kLbo128, kLbo128, 128), b, id, 1u);
            }
            mma_commit(&mb);
        }
        ok = wait_block(&mb, parity);
        parity ^= 1u;
        fence_after_sync();
        if (!ok) break;
    }

    // TMEM lane j holds feature f0 + j: columns 0..63 are its S_v row, 64 its z
    float* Wg = W + ((int64_t)bh * NG + g) * stride;
    if (ok) {
        const uint32_t ta = tbase + ((uint32_t)((warp & 3) * 32) << 16);
        float r[32];
        tmem_ld32(ta + half * 32, r);
        float zz[16];
        tmem_ld16(ta + kDV, zz);
        tmem_ld_wait();
        float4* so = reinterpret_cast<float4*>(sOut + row * L::kOutStride + half * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) so[i] = make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
        if (half == 1 && row < nf) Wg[(int64_t)F * kDV + f0 + row] = zz[0];
    } else {
        if (tid == 0) atomicOr(err, kErrPrefillPipe);
        ptx::mbar_wait(&mb, parity ^ 1u, kWaitPolls);  // one more bound for MMAs in flight
    }
    fence_before_sync();
    __syncthreads();
    if (ok) {
        float4* dst = reinterpret_cast<float4*>(Wg + (int64_t)f0 * kDV);
        for (int e = tid; e < nf * (kDV / 4); e += kThreads) {
            const int j = e / (kDV / 4), c = e % (kDV / 4);
            dst[e] = *reinterpret_cast<const float4*>(sOut + j * L::kOutStride + c * 4);
        }
    }
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tbase, 128);
    }
}

// ---------------------------------------------------------------- 3. outputs
template <int D>
struct OutSmem {
    static constexpr uint32_t kX = 0;                                  // q rows, fp32
    static constexpr uint32_t kQ = kX + XS<D>::kBytes;                 // Q, K-major 128 x D
    static constexpr uint32_t kU = kQ + kC * D * 2;                    // union of the two phases
    // pairwise phase
    static constexpr uint32_t kK = kU;                                 // K tile, K-major 128 x D
    static constexpr uint32_t kV1 = kK + kC * D * 2;                   // [V|1|0], MN-major K=128 x 80
    static constexpr uint32_t kPh = kV1 + kC * kNV * 2;                // P, K-major 128 x 128
    static constexpr uint32_t kPl = kPh + kC * kC * 2;
    static constexpr uint32_t kEndPair = kPl + kC * kC * 2;
    // read-out phase
    static constexpr uint32_t kAh = kU;                                // Phi_Q tile, K-major 128 x 128
    static constexpr uint32_t kAl = kAh + kC * kFT * 2;
    static constexpr uint32_t kSh = kAl + kC * kFT * 2;                // S tile, MN-major K=128 x 80
    static constexpr uint32_t kSl = kSh + kFT * kNV * 2;
    static constexpr uint32_t kEndRead = kSl + kFT * kNV * 2;
    static constexpr uint32_t kDesc = (kEndPair > kEndRead ? kEndPair : kEndRead);
    static constexpr uint32_t kBytes = kDesc + kFT * (uint32_t)sizeof(FeatDesc);
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
tcf_out_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k, const bf16* __restrict__ v,
               const float* __restrict__ W, float* __restrict__ out, int N, int n, float tau, int F,
               int64_t stride, int G, int NG, int carried, unsigned int* __restrict__ err) {
    using L = OutSmem<D>;
    extern __shared__ __align__(1024) uint8_t sm[];
    __shared__ __align__(8) uint64_t mb;
    __shared__ uint32_t tslot;
    __shared__ float qc[kMaxN];
    float* xs = reinterpret_cast<float*>(sm + L::kX);
    uint8_t* sQ = sm + L::kQ;
    uint8_t* sK = sm + L::kK;
    uint8_t* sV1 = sm + L::kV1;
    uint8_t* sPh = sm + L::kPh;
    uint8_t* sPl = sm + L::kPl;
    uint8_t* sAh = sm + L::kAh;
    uint8_t* sAl = sm + L::kAl;
    uint8_t* sSh = sm + L::kSh;
    uint8_t* sSl = sm + L::kSl;
    FeatDesc* ds = reinterpret_cast<FeatDesc*>(sm + L::kDesc);
    constexpr uint32_t kSboD = (uint32_t)(D / 8) * 128u;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int qt = blockIdx.x, bh = blockIdx.y;
    const int64_t q0 = (int64_t)qt * kC;
    const int nq = (int)min64(kC, (int64_t)N - q0);
    const int g = (int)(q0 / G);
    const int64_t gs = (int64_t)g * G;
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;
    const bool valid = row < nq;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;

    if (tid == 0) {
        ptx::mbar_init(&mb, 1);
        ptx::fence_mbar_init();
    }
    if (tid < n) qc[tid] = query_coeff(tid, tau);
    if (warp == 0) {
        tmem_alloc(&tslot, 256);
        tmem_relinquish();
    }
    const bf16* qb = q + ((int64_t)bh * N + q0) * D;
    stage_x<D>(xs, qb, nq);
    stage_kmajor_rows<D>(sQ, qb, nq);
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tA = tslot, tO = tslot + 128;

    bool ok = true;
    uint32_t phase = 0;
    bool first = true;
    // ------------------------------------------------ pairwise part, key tiles of this group
    for (int64_t k0 = gs; k0 <= q0 && ok; k0 += kC) {
        const int nk = (int)min64(kC, (int64_t)N - k0);
        stage_kmajor_rows<D>(sK, k + ((int64_t)bh * N + k0) * D, nk);
        stage_v1(sV1, v + ((int64_t)bh * N + k0) * kDV, nk, 10, kLboNV);
        publish_smem();
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks)
                mma_bf16(tA, smem_desc(sQ + ks * 256, 128, kSboD), smem_desc(sK + ks * 256, 128, kSboD), id,
                         ks > 0 ? 1u : 0u);
            mma_commit(&mb);
        }
        ok = wait_block(&mb, phase);
        phase ^= 1u;
        fence_after_sync();
        if (!ok) break;
        {
            float s0[32], s1[32];
            tmem_ld32(tA + lane_off + half * 64, s0);
            tmem_ld32(tA + lane_off + half * 64 + 32, s1);
            tmem_ld_wait();
            const bool diag = k0 == q0;
#pragma unroll
            for (int g8 = 0; g8 < 8; ++g8) {
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = g8 * 8 + e;
                    const int key = half * 64 + j;
                    const float x = tau * (j < 32 ? s0[j] : s1[j - 32]);
                    const bool keep = valid && key < nk && (!diag || key <= row);
                    p[e] = keep ? taylor_kernel(x, n) : 0.f;
                }
                uint4 hi, lo;
                split8(p, hi, lo);
                const int kg = half * 8 + g8;
                *reinterpret_cast<uint4*>(sPh + kmaj(row, kg, kSbo128)) = hi;
                *reinterpret_cast<uint4*>(sPl + kmaj(row, kg, kSbo128)) = lo;
            }
        }
        publish_smem();
        if (tid == 0) {
            const uint32_t id = idesc_bf16(128, kNV, 0, 1);
#pragma unroll
            for (int ks = 0; ks < kC / 16; ++ks) {
                const uint64_t b = smem_desc(sV1 + ks * 2 * kLboNV, kLboNV, 128);
                mma_bf16(tO, smem_desc(sPh + ks * 256, 128, kSbo128), b, id, (!first || ks > 0) ? 1u : 0u);
                mma_bf16(tO, smem_desc(sPl + ks * 256, 128, kSbo128), b, id, 1u);
            }
            mma_commit(&mb);
        }
        first = false;
        ok = wait_block(&mb, phase);
        phase ^= 1u;
        fence_after_sync();
    }

    // ------------------------------------------------ read-out through S_<g, feature tiles
    ptx::pdl_wait_primary();  // the scan over group states has completed
    if (ok && (g > 0 || carried)) {
        const float* Sg = W + ((int64_t)bh * NG + g) * stride;
        const int nft = (F + kFT - 1) / kFT;
        for (int ft = 0; ft < nft && ok; ++ft) {
            const int f0 = ft * kFT;
            load_tile_desc(ds, D, n, f0, F, tau, qc, true);
            // S tile rows f0.. as hi/lo, MN-major [K=128 features][80]
            for (int u = tid; u < kFT * 10; u += kThreads) {
                const int j = u / 10, gq = u % 10, f = f0 + j;
                float xv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (f < F) {
                    if (gq < 8) {
                        const float4 a = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + gq * 8));
                        const float4 b = __ldg(reinterpret_cast<const float4*>(Sg + (int64_t)f * kDV + gq * 8) + 1);
                        xv[0] = a.x; xv[1] = a.y; xv[2] = a.z; xv[3] = a.w;
                        xv[4] = b.x; xv[5] = b.y; xv[6] = b.z; xv[7] = b.w;
                    } else if (gq == 8) {
                        xv[0] = __ldg(Sg + (int64_t)F * kDV + f);
                    }
                }
                uint4 hi, lo;
                split8(xv, hi, lo);
                *reinterpret_cast<uint4*>(sSh + mnmaj(j, gq, kLboNV)) = hi;
                *reinterpret_cast<uint4*>(sSl + mnmaj(j, gq, kLboNV)) = lo;
            }
            __syncthreads();  // descriptors ready
            // Phi_Q[token row][features half*64 .. +64), K-major
            {
                const float* x = xs + row * XS<D>::kStride;
#pragma unroll
                for (int g8 = 0; g8 < 8; ++g8) {
                    const int j0 = half * 64 + g8 * 8;
                    float buf[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) buf[e] = valid ? eval_tile(ds[j0 + e], x) : 0.f;
                    uint4 hi, lo;
                    split8(buf, hi, lo);
                    *reinterpret_cast<uint4*>(sAh + kmaj(row, j0 / 8, kSbo128)) = hi;
                    *reinterpret_cast<uint4*>(sAl + kmaj(row, j0 / 8, kSbo128)) = lo;
                }
            }
            publish_smem();
            if (tid == 0) {
                const uint32_t id = idesc_bf16(128, kNV, 0, 1);
#pragma unroll
                for (int ks = 0; ks < kFT / 16; ++ks) {
                    const uint64_t ah = smem_desc(sAh + ks * 256, 128, kSbo128);
                    const uint64_t al = smem_desc(sAl + ks * 256, 128, kSbo128);
                    const uint64_t bh_ = smem_desc(sSh + ks * 2 * kLboNV, kLboNV, 128);
                    const uint64_t bl_ = smem_desc(sSl + ks * 2 * kLboNV, kLboNV, 128);
                    mma_bf16(tO, ah, bh_, id, 1u);
                    mma_bf16(tO, ah, bl_, id, 1u);
                    mma_bf16(tO, al, bh_, id, 1u);
                }
                mma_commit(&mb);
            }
            ok = wait_block(&mb, phase);
            phase ^= 1u;
            fence_after_sync();
        }
    }

    // ------------------------------------------------ epilogue
    if (ok) {
        float o[32], dn[16];
        tmem_ld32(tO + lane_off + half * 32, o);
        tmem_ld16(tO + lane_off + kDV, dn);
        tmem_ld_wait();
        if (valid) {
            const float r = __frcp_rn(dn[0]);
            float4* dst = reinterpret_cast<float4*>(out + ((int64_t)bh * N + q0 + row) * kDV + half * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(o[4 * i] * r, o[4 * i + 1] * r, o[4 * i + 2] * r, o[4 * i + 3] * r);
        }
    } else {
        if (tid == 0) atomicOr(err, kErrPrefillPipe);
        ptx::mbar_wait(&mb, phase ^ 1u, kWaitPolls);  // one more bound for MMAs in flight
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tslot, 256);
    }
}

constexpr int kMaxDevices = 64;

template <int D>
int run(const bf16* q, const bf16* k, const bf16* v, float* out, const float* state_in, float* state_out, int BH,
        int N, int n, float tau, int64_t F, int64_t stride, unsigned int* err, cudaStream_t stream) {
    static std::once_flag once[kMaxDevices];
    static cudaError_t res[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TAYLOR_ERR_CUDA;
    std::call_once(once[dev], [&]() {
        res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_state_kernel<D>),
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StateSmem<D>::kBytes);
        if (res[dev] == cudaSuccess)
            res[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(tcf_out_kernel<D>),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)OutSmem<D>::kBytes);
    });
    if (res[dev] != cudaSuccess) return TAYLOR_ERR_CUDA;

    // group size: pairwise work G (d + 160) per token against 480 F per token
    // for the read-out, within [128, 2048] and no larger than the sequence
    int G = 128;
    while (G < 2048 && (int64_t)G * (D + 160) < 240 * F) G *= 2;
    while (G > 128 && G / 2 >= N) G /= 2;
    const int NG = (N + G - 1) / G;
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
                 tcf_state_kernel<D><<<dim3(NG, NFT, BH), kThreads, StateSmem<D>::kBytes, stream>>>(
                     k, v, Wb, N, n, (int)F, stride, G, NG, err));
        e = cudaGetLastError();
        if (e == cudaSuccess) e = launch_state_scan(Wb, state_in, state_out, BH, NG, stride, F * (kDV + 1), stream, true);
    }
    if (e == cudaSuccess) {
        const int NQ = (N + kC - 1) / kC;
        TA_TIMED(stream, "tcf_out_kernel",
                 e = launch_maybe_pdl(tcf_out_kernel<D>, dim3(NQ, BH), dim3(kThreads), OutSmem<D>::kBytes, stream,
                                      need_ws, q, k, v, (const float*)Wb, out, N, n, tau, (int)F, stride, G, NG,
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

}  // namespace

int try_prefill_tiled(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream) {
    if (dv != kDV || N <= 0 || BH <= 0) return kNotApplicable;
    unsigned int* err = device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;
    switch (d) {
        case 16: return run<16>(q, k, v, out, state_in, state_out, BH, N, n, tau, F, stride, err, stream);
        case 32: return run<32>(q, k, v, out, state_in, state_out, BH, N, n, tau, F, stride, err, stream);
        case 64: return run<64>(q, k, v, out, state_in, state_out, BH, N, n, tau, F, stride, err, stream);
        default: return kNotApplicable;
    }
}

}  // namespace tc
}  // namespace ta
