// Batched multi-token decode with the contractions on the tensor cores: T <= 16
// new tokens per head against the head's carried state, for bf16 q, k, v,
// d_v = 64 and at most 160 features of degree <= 2 (d_k = 16 at n = 3).
// What it computes is the decode step of the paper (arXiv 2610.20637,
// abstract: constant per-token cost, the history held in the additive states)
// for a block of tokens, with the block's own causal part pairwise:
//   num_i = (c (.) phi(q_i))^T S + sum_{j <= i} K(q_i, k_j) v_j,
//   den_i = (c (.) phi(q_i))^T z + sum_{j <= i} K(q_i, k_j),   o_i = num_i / den_i,
//   S' = S + sum_j phi(k_j) v_j^T,   z' = z + sum_j phi(k_j).
//
// Per head, two tcgen05 contractions (one thread issues them, fp32 in TMEM):
//  * the update, D_U[f][c'] = sum_j phi_f(k_j) [v_j | 1][c']: A = phi(k) split
//    as hi + lo bf16 (two MMAs a 128-feature tile, M 128 x N 80 x K 16), B = V
//    (bf16, exact) with a column of ones after it, whose column gives z's
//    increment;
//  * the read-out, D_R[c][i] = sum_f S[f][c] c_f phi_f(q_i) + sum_j v_j[c] P[i][j]:
//    one MMA a K step (M 128 x N 32 x K 16) with A = [S_hi | S_lo] (MN-major:
//    v column c is row c of D, its lo part row 64 + c) and B = the query
//    features [hi | lo] (tokens 0..15, then 16..31), so that D holds all
//    four products hi.hi, hi.lo, lo.hi, lo.lo; then A = [V | 0] against the
//    pairwise weights [P_hi | P_lo].
// The state arrives by TMA as two fp32 slabs (columns 0..31 and 32..63) of
// 128-byte rows with the 128-byte swizzle.  In the update epilogue the thread
// of feature row f (its TMEM lane) reads its row without bank conflicts into
// registers and writes S'[f] = S[f] + D_U[f] back in its place; two TMA
// tensor stores take the slabs to HBM (unswizzled by the copy engine, whole
// lines).  Once they have read the slabs, each thread writes the bf16 hi and
// lo images of its old row over the same two 128-byte rows: in the
// read-out's MN-major 128-byte-swizzled layout row f of S_hi sits exactly
// where slab 0's row f is, and row f of S_lo where slab 1's is.  The
// normalisers are CUDA-core sums on the side.
//
// Three ring buffers (state, z, q, k, v rows of one head) serve two
// warpgroups that take the CTA's heads in turn; the warpgroup done with head
// i issues head i + 3 into the buffer it frees.  state_out may alias
// state_in.  HBM traffic is one state read and one state write per head, as
// for a single decode step.
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"
#include "phase.cuh"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tmap.h"

namespace ta {

namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kTT = 16;    // tokens per call, padded
constexpr int kFT = 160;   // features, padded
constexpr int kDVt = 64;
constexpr int kWGt = 2, kWGtThreads = 128, kThreadsT = kWGt * kWGtThreads;
constexpr int kNBuf = 3;
constexpr uint32_t kPolls = 1u << 22;
constexpr uint32_t kHalfS = kFT * 128;  // bytes of one bf16 image of the state (S_hi, then S_lo)
constexpr size_t kMaxDynT = 226 * 1024;
constexpr int kMaxDevicesT = 64;

struct TcLayout {
    uint32_t offz, offq, offk, offv, buf;                // one ring buffer
    uint32_t v2, pk, pq, pt, qf, kf, zp, ps, den, area;  // one warpgroup area
    uint32_t areas, desc, bytes;
};

__host__ __device__ inline uint32_t al128(uint32_t x) { return (x + 127u) & ~127u; }
__host__ __device__ inline uint32_t al1k(uint32_t x) { return (x + 1023u) & ~1023u; }

// z's bulk copy: F floats rounded up to 16 bytes
__host__ __device__ inline uint32_t z_bytes(int F) { return (uint32_t)((F * 4 + 15) & ~15); }

__host__ __device__ inline TcLayout tc_layout(int T, int d, int F) {
    TcLayout L;
    // [0, 2 kHalfS): the fp32 slabs (F rows of 128 bytes at 0 and kHalfS),
    // later S_hi and S_lo (160 rows of 128 bytes each, same places)
    L.offz = 2 * kHalfS;
    L.offq = L.offz + al128(z_bytes(F));
    L.offk = L.offq + al128((uint32_t)(T * d) * 2);
    L.offv = L.offk + al128((uint32_t)(T * d) * 2);
    L.buf = al1k(L.offv + (uint32_t)(T * kDVt) * 2);
    L.v2 = 0;                       // V, a column of ones, zeros: MN-major 128-byte swizzle, 3 atoms of 2 KB
    L.pk = 6144;                    // phi(k) hi, lo: K-major, [f/8][j/8][f%8][j%8], 2 x 5 KB; later the read-out's lo rows
    L.pq = L.pk + 2 * 5120;         // query features: K-major, [f/8][i'/8][i'%8][f%8], i' = i (hi), 16 + i (lo), 10 KB
    L.pt = L.pq + 2 * 5120;         // pairwise weights: K-major, [j/8][i'/8][i'%8][j%8], 1 KB
    L.qf = L.pt + 1024;             // q, k rows in fp32 with a slot of 1: [16][d + 1]
    L.kf = L.qf + al128((uint32_t)(kTT * (d + 1)) * 4);
    L.zp = L.kf + al128((uint32_t)(kTT * (d + 1)) * 4);  // query features . z over feature quads: [40][16]
    L.ps = L.zp + 40 * kTT * 4;     // sum_j P[i][j]: [16]
    L.den = L.ps + kTT * 4;         // reciprocal normalisers: [16]
    L.area = al1k(L.den + kTT * 4);
    L.areas = kNBuf * L.buf;
    L.desc = L.areas + kWGt * L.area;  // [160] float4: {a | c << 8, w, w tau^m/m!, 0}
    L.bytes = L.desc + kFT * 16 + 1024;  // + alignment slack
    return L;
}

__device__ __forceinline__ unsigned char* align_1k(unsigned char* p) {
    const uint32_t a = ptx::smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void wg_sync(int wg) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + wg), "r"(kWGtThreads) : "memory");
}

// Byte offset of 16-byte chunk ch of row r in rows of 128 bytes with the
// 128-byte swizzle (1024-byte aligned base).
__device__ __forceinline__ uint32_t sw128(int r, int ch) {
    return (uint32_t)r * 128u + ((uint32_t)(ch ^ (r & 7)) << 4);
}

struct MultiTcArgs {
    const bf16* q;
    const bf16* k;
    const bf16* v;
    const float* state_in;
    float* state_out;
    float* out;
    unsigned int* err;
    int64_t stride;
    int BH, T, d, n, F;
    float tau;
};

// Feature row f of the state from its two fp32 slab rows (zeros if not live).
__device__ __forceinline__ void load_row(const unsigned char* buf, int f, bool live, float (&s)[64]) {
#pragma unroll
    for (int p = 0; p < 16; ++p) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (live) x = *reinterpret_cast<const float4*>(buf + (p >> 3) * kHalfS + sw128(f, p & 7));
        s[4 * p] = x.x; s[4 * p + 1] = x.y; s[4 * p + 2] = x.z; s[4 * p + 3] = x.w;
    }
}

// The bf16 hi and lo images of row f over its slab rows (slab 0 takes hi,
// slab 1 lo); the thread has read the whole row before.
__device__ __forceinline__ void image_row(unsigned char* buf, int f, const float (&s)[64]) {
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        uint4 hi, lo;
        split8(s + 8 * b, hi, lo);
        *reinterpret_cast<uint4*>(buf + sw128(f, b)) = hi;
        *reinterpret_cast<uint4*>(buf + kHalfS + sw128(f, b)) = lo;
    }
}

// The update epilogue of feature row f (this thread's TMEM lane in the tile
// at column tcol), once the read-out has finished with the images:
// S'[f] = S[f] + D_U[f][0..63] into the slab rows, z'_f = z_f + D_U[f][64] to HBM.
__device__ __forceinline__ void update_row(unsigned char* buf, const float* Z, float* G, int F, int f, bool live,
                                           uint32_t tcol, const float (&s)[64]) {
    float dl[64];
    tmem_ld32(tcol, *reinterpret_cast<float(*)[32]>(dl));
    tmem_ld32(tcol + 32, *reinterpret_cast<float(*)[32]>(dl + 32));
    const float dz = tmem_ld1(tcol + 64);
    tmem_ld_wait();
    if (!live) return;
#pragma unroll
    for (int p = 0; p < 16; ++p)
        *reinterpret_cast<float4*>(buf + (p >> 3) * kHalfS + sw128(f, p & 7)) =
            make_float4(s[4 * p] + dl[4 * p], s[4 * p + 1] + dl[4 * p + 1], s[4 * p + 2] + dl[4 * p + 2],
                        s[4 * p + 3] + dl[4 * p + 3]);
    if (G) G[(int64_t)F * kDVt + f] = Z[f] + dz;
}

__global__ void __launch_bounds__(kThreadsT, 1)
decode_multi_tc_kernel(const __grid_constant__ CUtensorMap tms, const __grid_constant__ CUtensorMap tmo,
                       const MultiTcArgs A) {
    extern __shared__ __align__(1024) unsigned char dsm_raw[];
    unsigned char* dsm = align_1k(dsm_raw);
    __shared__ __align__(8) uint64_t full[kNBuf], mma_u[kWGt], mma_r[kWGt];
    __shared__ uint32_t s_tmem;
    __shared__ int s_bad, s_fail[kWGt];
    __shared__ volatile int s_issued[kNBuf];  // the head last issued into each buffer
    const int T = A.T, d = A.d, F = A.F;
    const TcLayout L = tc_layout(T, d, F);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nheads = A.BH > (int)blockIdx.x ? (A.BH - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    const int nks = (F + 15) >> 4, NF = 16 * nks, ntiles = NF > 128 ? 2 : 1;
    const uint32_t tok_in = (uint32_t)(T * d) * 2u, tok_v = (uint32_t)(T * kDVt) * 2u, zb = z_bytes(F);
    auto issue = [&](int i) {  // head i of this CTA into buffer i mod 3 (one thread)
        const int b = i % kNBuf;
        const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
        unsigned char* buf = dsm + (size_t)b * L.buf;
        ptx::mbar_arrive_expect_tx(&full[b], 2u * (uint32_t)F * 128u + zb + 2 * tok_in + tok_v);
        ptx::tma_load_3d(buf, &tms, 0, 0, (int)h, &full[b]);
        ptx::tma_load_3d(buf + kHalfS, &tms, 32, 0, (int)h, &full[b]);
        ptx::bulk_g2s(buf + L.offz, A.state_in + h * A.stride + (int64_t)F * kDVt, zb, &full[b]);
        ptx::bulk_g2s(buf + L.offq, A.q + h * T * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + L.offk, A.k + h * T * d, tok_in, &full[b]);
        ptx::bulk_g2s(buf + L.offv, A.v + h * T * kDVt, tok_v, &full[b]);
        s_issued[b] = i;
    };

    // launched with programmatic dependent launch: every global memory access
    // of the grid follows thread 0's wait on the previous grid (directly, or
    // through the barrier below)
    ptx::pdl_launch_dependents();
    if (tid == 0) {
        for (int i = 0; i < kNBuf; ++i) {
            ptx::mbar_init(&full[i], 1);
            s_issued[i] = -1;
        }
        for (int i = 0; i < kWGt; ++i) {
            ptx::mbar_init(&mma_u[i], 1);
            ptx::mbar_init(&mma_r[i], 1);
        }
        ptx::fence_mbar_init();
        ptx::pdl_wait_primary();
        for (int i = 0; i < kNBuf && i < nheads; ++i) issue(i);
        s_bad = 0;
    }
    if (tid < kWGt) s_fail[tid] = 0;
    if (warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    // the feature table: indices (d for a missing factor, which reads the
    // slot of 1 after each q, k row) and both weights
    float4* desc = reinterpret_cast<float4*>(dsm + L.desc);
    for (int f = tid; f < F; f += kThreadsT) {
        int m, a, c2;
        float w;
        feature_deg2(d, f, m, a, c2, w);
        if (m < 2) c2 = d;
        if (m < 1) a = d;
        desc[f] = make_float4(__int_as_float(a | (c2 << 8)), w, w * query_coeff(m, A.tau), 0.f);
    }
    // rows F..NF-1 of the state images stay zero (no copy writes them), and
    // each warpgroup's second B atom of the update is a column of ones
    for (int e = tid; e < kNBuf * 2 * (NF - F) * 8; e += kThreadsT) {
        const int b = e / (2 * (NF - F) * 8), r = e % (2 * (NF - F) * 8);
        const int half = r / ((NF - F) * 8), rr = r % ((NF - F) * 8);
        *reinterpret_cast<uint4*>(dsm + (size_t)b * L.buf + half * kHalfS + (uint32_t)(F + rr / 8) * 128u +
                                  (uint32_t)(rr % 8) * 16u) = make_uint4(0, 0, 0, 0);
    }
    for (int e = tid; e < kWGt * 256; e += kThreadsT) {  // the ones atom, then the zero atom: 128 chunks each
        const int w = e >> 8, at = (e >> 7) & 1, ch = e & 127, j = ch >> 3, c = ch & 7;  // K row j (16), chunk c
        uint4 val = make_uint4(0, 0, 0, 0);
        if (at == 0 && c == (j & 7)) val.x = 0x3F80u;  // bf16 1.0 in column 0: chunk 0, swizzled to chunk j % 8
        *reinterpret_cast<uint4*>(dsm + L.areas + (size_t)w * L.area + L.v2 + 2048 * (1 + at) +
                                  (uint32_t)(j >> 3) * 1024u + (uint32_t)(j & 7) * 128u + (uint32_t)c * 16u) = val;
    }
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();

    const float tau = A.tau;
    const int n = A.n;
    const int wg = warp >> 2, t = tid & (kWGtThreads - 1), wl = warp & 3;
    unsigned char* area = dsm + L.areas + (size_t)wg * L.area;
    unsigned char* v2 = area + L.v2;
    unsigned char* pkh = area + L.pk;
    unsigned char* pkl = pkh + 5120;
    unsigned char* pq = area + L.pq;
    unsigned char* pt = area + L.pt;
    float* rlo = reinterpret_cast<float*>(area + L.pk);  // [16][64], after the update MMAs
    float* qf = reinterpret_cast<float*>(area + L.qf);
    float* kf = reinterpret_cast<float*>(area + L.kf);
    float* zp = reinterpret_cast<float*>(area + L.zp);
    float* ps = reinterpret_cast<float*>(area + L.ps);
    float* rden = reinterpret_cast<float*>(area + L.den);
    const uint32_t tU = s_tmem + 256u * (uint32_t)wg, tR = tU + 160u;
    const uint32_t lane_off = (uint32_t)(32 * wl) << 16;
    TA_PHASE_VARS(p_t, p_wait = 0, p_prep = 0, p_upd = 0, p_conv = 0, p_ro = 0);
    int kh = 0;  // heads done by this warpgroup: the parity of its MMA barriers
    for (int i = wg; i < nheads; i += kWGt, ++kh) {
        const int b = i % kNBuf;
        TA_PHASE_T0(p_t);
        // head i's copies are issued only after head i - 3 has left the
        // buffer, so once s_issued says so the barrier's pending phase is head i's
        bool ok = true;
        for (uint32_t it = 0; s_issued[b] != i; ++it)
            if (it > kPolls || s_bad) {
                ok = false;
                break;
            }
        if (!ok || !ptx::mbar_wait_or_abort(&full[b], (uint32_t)(i / kNBuf) & 1u, kPolls, &s_bad)) s_fail[wg] = 1;
        wg_sync(wg);
        if (s_fail[wg]) break;  // the same value for all 128 threads: set only before this barrier
        TA_PHASE_ACC(p_wait, p_t);
        TA_PHASE_T0(p_t);
        const int64_t h = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
        unsigned char* buf = dsm + (size_t)b * L.buf;
        const float* Z = reinterpret_cast<const float*>(buf + L.offz);
        const bf16* xq = reinterpret_cast<const bf16*>(buf + L.offq);
        const bf16* xk = reinterpret_cast<const bf16*>(buf + L.offk);
        const bf16* xv = reinterpret_cast<const bf16*>(buf + L.offv);

        // (1) q, k rows in fp32 with the slot of 1 (rows T..15 all ones); V
        // into the first swizzled atom (rows T..15 zero)
        {
            const int j = t >> 3;  // 8 threads a token row
            const bool live = j < T;
            for (int c = t & 7; c <= d; c += 8) {
                qf[j * (d + 1) + c] = c < d && live ? __bfloat162float(xq[j * d + c]) : 1.f;
                kf[j * (d + 1) + c] = c < d && live ? __bfloat162float(xk[j * d + c]) : 1.f;
            }
            const int ch = t & 7;
            const uint4 val = live ? *reinterpret_cast<const uint4*>(xv + j * kDVt + 8 * ch) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(v2 + (uint32_t)(j >> 3) * 1024u + sw128(j & 7, ch)) = val;
        }
        wg_sync(wg);

        // (2) the coefficient operands, hi and lo
        // phi(k): one thread per (feature f, tokens 4 j4 .. 4 j4 + 3)
        for (int u = t; u < NF * 4; u += kWGtThreads) {
            const int f = u >> 2, j4 = u & 3;
            const float4 fd = desc[f < F ? f : 0];
            const int a = __float_as_int(fd.x) & 255, c2 = __float_as_int(fd.x) >> 8;
            const float wf = f < F ? fd.y : 0.f;
            float kk[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * j4 + jj;
                const float* kr = kf + j * (d + 1);  // rows T..15 hold finite values
                kk[jj] = (j < T ? wf : 0.f) * kr[a] * kr[c2];
            }
            uint2 hi, lo;
            split2(kk[0], kk[1], hi.x, lo.x);
            split2(kk[2], kk[3], hi.y, lo.y);
            const uint32_t off = (uint32_t)(f >> 3) * 256u + (uint32_t)(j4 >> 1) * 128u + (uint32_t)(f & 7) * 16u +
                                 (uint32_t)(j4 & 1) * 8u;
            *reinterpret_cast<uint2*>(pkh + off) = hi;
            *reinterpret_cast<uint2*>(pkl + off) = lo;
        }
        // query features: one thread per (token i, features 4 g .. 4 g + 3),
        // with the partial normaliser sum_f c_f phi_f(q_i) z_f
        for (int u = t; u < kTT * 4 * nks; u += kWGtThreads) {
            const int i2 = u & 15, g = u >> 4;
            const float* qr = qf + i2 * (d + 1);  // rows T..15 hold finite values
            float4 fd[4];
            float zf[4], x[4], zs = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int f = 4 * g + r;
                fd[r] = desc[f < F ? f : 0];
                zf[r] = Z[f < F ? f : 0];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int f = 4 * g + r;
                const int a = __float_as_int(fd[r].x) & 255, c2 = __float_as_int(fd[r].x) >> 8;
                x[r] = (f < F && i2 < T ? fd[r].z : 0.f) * qr[a] * qr[c2];
                zs = fmaf(x[r], zf[r], zs);
            }
            uint2 hi, lo;
            split2(x[0], x[1], hi.x, lo.x);
            split2(x[2], x[3], hi.y, lo.y);
            const uint32_t off = (uint32_t)(g >> 1) * 512u + (uint32_t)(i2 >> 3) * 128u + (uint32_t)(i2 & 7) * 16u +
                                 (uint32_t)(g & 1) * 8u;
            *reinterpret_cast<uint2*>(pq + off) = hi;
            *reinterpret_cast<uint2*>(pq + 256 + off) = lo;  // rows 16 + i
            zp[g * kTT + i2] = zs;
        }
        // the block's pairwise weights K(tau q_i.k_j), j <= i: one thread per
        // (token i, tokens 2 jp, 2 jp + 1), with the row sums
        {
            const int i2 = t >> 3, j0 = 2 * (t & 7);
            float pw[2] = {0.f, 0.f};
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                if (i2 < T && j0 + u <= i2) {
                    float dot = 0.f;
                    for (int c = 0; c < d; ++c) dot = fmaf(qf[i2 * (d + 1) + c], kf[(j0 + u) * (d + 1) + c], dot);
                    pw[u] = taylor_kernel(tau * dot, n);
                }
            }
            uint32_t hi, lo;
            split2(pw[0], pw[1], hi, lo);
            const uint32_t off = (uint32_t)(j0 >> 3) * 512u + (uint32_t)(i2 >> 3) * 128u + (uint32_t)(i2 & 7) * 16u +
                                 (uint32_t)(j0 & 7) * 2u;
            *reinterpret_cast<uint32_t*>(pt + off) = hi;
            *reinterpret_cast<uint32_t*>(pt + 256 + off) = lo;  // rows 16 + i
            float s = pw[0] + pw[1];
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if ((t & 7) == 0) ps[i2] = s;
        }
        ptx::fence_proxy_async_smem();  // the operands, for the tensor cores
        fence_before_sync();
        wg_sync(wg);
        TA_PHASE_ACC(p_prep, p_t);
        TA_PHASE_T0(p_t);

        // (3) every thread takes its feature row(s) of the state into registers
        // and writes their bf16 images in place for the read-out
        float s0[64], s1[64];
        const int f0 = 32 * wl + lane, f1 = 128 + lane;
        const bool two = ntiles > 1 && wl == 0;  // tile 1 (features 128..255) lies in lanes 0..31 too
        load_row(buf, f0, f0 < F, s0);
        if (two) load_row(buf, f1, f1 < F, s1);
        if (f0 < F) image_row(buf, f0, s0);
        if (two && f1 < F) image_row(buf, f1, s1);
        ptx::fence_proxy_async_smem();
        fence_before_sync();
        wg_sync(wg);
        TA_PHASE_ACC(p_upd, p_t);
        TA_PHASE_T0(p_t);

        // (4) both contractions on the tensor cores
        if (t == 0) {
            fence_after_sync();
            // the update, D_U[f][c'] = sum_j phi_f(k_j) [v_j | 1][c']
            const uint64_t bv = smem_desc_sw(v2, 2048, 1024, kSwizzle128);
            const uint32_t iu = idesc_bf16(128, 80, 0, 1);
            for (int x = 0; x < ntiles; ++x) {
                mma_bf16(tU + 80u * (uint32_t)x, smem_desc(pkh + 4096 * x, 128, 256), bv, iu, 0);
                mma_bf16(tU + 80u * (uint32_t)x, smem_desc(pkl + 4096 * x, 128, 256), bv, iu, 1);
            }
            // the read-out, A = [S_hi | S_lo] (the second 64-row atom, through
            // LBO, is the lo image) against [Q_hi | Q_lo]; step s starts 2048 (A)
            // and 1024 (B) bytes on, added to the address fields (>> 4)
            const uint32_t ir = idesc_bf16(128, 2 * kTT, 1, 0);
            const uint64_t as = smem_desc_sw(buf, kHalfS, 1024, kSwizzle128);
            const uint64_t bq = smem_desc(pq, 512, 128);
            for (int s = 0; s < nks; ++s)
                mma_bf16(tR, as + (uint64_t)(128 * s), bq + (uint64_t)(64 * s), ir, s > 0 ? 1u : 0u);
            // A = [V | 0] (the zero atom as rows 64..127) against [P_hi | P_lo]
            mma_bf16(tR, smem_desc_sw(v2, 4096, 1024, kSwizzle128), smem_desc(pt, 512, 128), ir, 1);
            mma_commit(&mma_u[wg]);
        }
        // meanwhile: the normalisers (their reciprocals), the state's padding
        float* G = A.state_out ? A.state_out + h * A.stride : nullptr;
        {
            const int i2 = t >> 3, g0 = t & 7;  // 8 threads a token
            float sm = g0 == 0 ? ps[i2] : 0.f;
            for (int g = g0; g < 4 * nks; g += 8) sm += zp[g * kTT + i2];
            sm += __shfl_xor_sync(0xffffffffu, sm, 1);
            sm += __shfl_xor_sync(0xffffffffu, sm, 2);
            sm += __shfl_xor_sync(0xffffffffu, sm, 4);
            if (g0 == 0) rden[i2] = 1.f / sm;
        }
        if (G)
            for (int64_t e = (int64_t)F * (kDVt + 1) + t; e < A.stride; e += kWGtThreads) G[e] = 0.f;
        if (!ptx::mbar_wait(&mma_u[wg], (uint32_t)kh & 1u, kPolls)) s_bad = 1;
        fence_after_sync();
        TA_PHASE_ACC(p_conv, p_t);
        TA_PHASE_T0(p_t);

        // (5) the update epilogue, feature row by row (TMEM lane = row): the
        // images are no longer read, S' replaces them; the read-out's lo rows
        update_row(buf, Z, G, F, f0, f0 < F, tU + lane_off, s0);
        if (two) update_row(buf, Z, G, F, f1, f1 < F, tU + 80u + lane_off, s1);
        float y[32];
        tmem_ld32(tR + lane_off, y);
        tmem_ld_wait();
        const int col = (32 * wl + lane) & 63;
        if (wl >= 2) {
#pragma unroll
            for (int i2 = 0; i2 < kTT; ++i2) rlo[i2 * kDVt + col] = y[i2] + y[kTT + i2];
        }
        ptx::fence_proxy_async_smem();  // S' in the slabs, for the tensor stores
        fence_before_sync();
        wg_sync(wg);
        if (t == 0 && G) {
            ptx::tma_store_3d(&tmo, 0, 0, (int)h, buf);
            ptx::tma_store_3d(&tmo, 32, 0, (int)h, buf + kHalfS);
            ptx::bulk_commit();
        }
        // (6) the outputs: hi rows (warps 0, 1) plus the lo rows, times 1 / den
        if (wl < 2) {
#pragma unroll
            for (int i2 = 0; i2 < kTT; ++i2)
                if (i2 < T) A.out[(h * T + i2) * kDVt + col] = (y[i2] + y[kTT + i2] + rlo[i2 * kDVt + col]) * rden[i2];
        }
        fence_before_sync();
        wg_sync(wg);
        TA_PHASE_ACC(p_ro, p_t);
        // (7) once the tensor stores have read the slabs the buffer is free:
        // bring in head i + 3
        if (t == 0 && i + kNBuf < nheads) {
            ptx::bulk_wait_read_all();
            issue(i + kNBuf);
        }
    }
    TA_PHASE_PUT(0, 1 + 5 * wg, tid == 128 * wg, p_wait);
    TA_PHASE_PUT(0, 2 + 5 * wg, tid == 128 * wg, p_prep);
    TA_PHASE_PUT(0, 3 + 5 * wg, tid == 128 * wg, p_upd);
    TA_PHASE_PUT(0, 4 + 5 * wg, tid == 128 * wg, p_conv);
    TA_PHASE_PUT(0, 5 + 5 * wg, tid == 128 * wg, p_ro);
    if ((tid & (kWGtThreads - 1)) == 0) ptx::bulk_wait_all();  // the state stores have completed
    fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        // copies still in flight after a failure must land before the block exits
        for (int b = 0; b < kNBuf; ++b) {
            const int i = s_issued[b];
            if (i >= 0) ptx::mbar_wait(&full[b], (uint32_t)(i / kNBuf) & 1u, kPolls);
        }
        if (s_bad) atomicOr(A.err, kErrDecodeLoad);
    }
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(s_tmem, 512);
    }
}

}  // namespace

cudaError_t launch_decode_multi_tc(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v,
                                   const float* state_in, float* state_out, float* out, int BH, int T, int d, int dv,
                                   int n, float tau, int64_t F, int64_t stride, cudaStream_t stream) {
    if (dv != kDVt || F > kFT || F < 1 || n > 3 || d > 32 || T < 1 || T > kTT || ((int64_t)T * d * 2) % 16 != 0)
        return cudaErrorNotSupported;
    // z's copy reads up to 3 floats of the state's padding; TMA wants 16-byte strides and base
    if ((int64_t)F * kDVt * 4 + z_bytes((int)F) > stride * 4 || (stride * 4) % 16 != 0 ||
        (reinterpret_cast<uintptr_t>(state_in) & 15) != 0)
        return cudaErrorNotSupported;
    static std::once_flag once[kMaxDevicesT];
    static cudaError_t set_err[kMaxDevicesT];
    static int num_sms[kMaxDevicesT];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevicesT) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [&]() {
        set_err[dev] = cudaFuncSetAttribute(reinterpret_cast<const void*>(decode_multi_tc_kernel),
                                            cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxDynT);
        if (set_err[dev] == cudaSuccess)
            set_err[dev] = cudaDeviceGetAttribute(&num_sms[dev], cudaDevAttrMultiProcessorCount, dev);
    });
    if (set_err[dev] != cudaSuccess) return set_err[dev];
    if (BH < 2 * num_sms[dev]) return cudaErrorNotSupported;  // few heads: one CTA per head is as good
    const TcLayout L = tc_layout(T, d, (int)F);
    if (L.bytes > kMaxDynT) return cudaErrorNotSupported;
    unsigned int* err = device_error_word();
    if (!err) return cudaErrorNotSupported;
    // the state as [BH][F rows][64] fp32 with row stride 256 bytes, read in
    // two slabs of 32 columns (128-byte rows, 128-byte swizzle)
    CUtensorMap tms, tmo;
    if (make_tmap_f32_3d(&tms, state_in, kDVt, (uint64_t)F, (uint64_t)BH, kDVt * 4, (uint64_t)stride * 4, 32,
                         (uint32_t)F, 128) != cudaSuccess)
        return cudaErrorNotSupported;
    if (state_out && ((reinterpret_cast<uintptr_t>(state_out) & 15) != 0 ||
                      make_tmap_f32_3d(&tmo, state_out, kDVt, (uint64_t)F, (uint64_t)BH, kDVt * 4,
                                       (uint64_t)stride * 4, 32, (uint32_t)F, 128) != cudaSuccess))
        return cudaErrorNotSupported;
    if (!state_out) tmo = tms;  // not used
    MultiTcArgs args{q, k, v, state_in, state_out, out, err, stride, BH, T, d, n, (int)F, tau};
    const int grid = num_sms[dev] < BH ? num_sms[dev] : BH;
    cudaError_t e = cudaSuccess;
    TA_TIMED(stream, "decode_multi_tc_kernel",
             e = launch_maybe_pdl(decode_multi_tc_kernel, dim3(grid), dim3(kThreadsT), (size_t)L.bytes, stream, true,
                                  tms, tmo, args));
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace ta
