// Causal prefill in one kernel launch on the sm_100a tensor cores, for d_k =
// 16, n <= 3 (F <= 153, padded to 160), d_v = 64, bf16 inputs, when every
// CTA of the call (one or two 128-token chunks each) can be resident at once.
//
// Method (arXiv 2610.20637, abstract): the causal history is the state
// S = sum_j phi(k_j) [v_j | 1]^T, additive across chunks, so prefill is a
// scan over chunk states.  CTA s of head h takes chunks a = NCH s and, when
// NCH = 2, b = a + 1:
//   1. loads its q, k, v rows with TMA (swizzled operand layouts);
//   2. forms its state T_s^T = sum_x [V_x | 1 | 0]^T Phi_K,x on the tensor
//      cores (TMEM, both chunks into one accumulator) and publishes it to
//      global memory (L2): staged in shared memory, one bulk store by the
//      publishing warp, then the head's count of published states is raised;
//   3. meanwhile forms the pairwise parts O_a = (poly(tau Q_a K_a^T) (.) mask) [V_a | 1],
//      O_b likewise with chunk b's own keys, plus all of chunk a's keys
//      (no mask): chunk b's view of chunk a is pairwise, not through a state;
//   4. the scan: the CTA that owns feature rows [R s, R s + R) of head h
//      (R = ceil(F / CTAs of the head)) waits for every state of the head,
//      gathers those rows of all of them into shared memory with bulk
//      copies, forms the exclusive prefixes E_s = state_in + sum_{s' < s} T_s'
//      for every CTA s of the head, and writes them, split into hi/lo bf16,
//      straight in the byte layout of the read-out MMA's operand (and the
//      total into state_out), then raises the head's count of scanned rows;
//   5. once that count reaches F, the CTA pulls its operand E_s with a bulk
//      copy, evaluates c (.) Phi_Q,x into TMEM and adds (c (.) Phi_Q,x) E_s to
//      O_x of both its chunks; o = O[:, :64] / O[:, 64], staged in shared
//      memory and written by TMA tensor stores.
// The launch is cooperative, so all CTAs that wait on one another's flags are
// resident together; every flag wait and every mbarrier wait is bounded, and
// a wait that runs out sets a device error bit and skips the work that
// depended on it.
//
// Precision as in the other tensor-core prefill: every operand produced in
// fp32 (Phi_K, Phi_Q, the pairwise weights P, the carried state E) is split
// into hi = x truncated to bf16 and lo = bf16(x - hi) and contracted as
// hi*hi' + hi*lo' + lo*hi' (or hi*B + lo*B against an exact bf16 input),
// fp32 accumulation.
//
// Roles: warps 0-7 (two per TMEM lane quadrant; thread = token or query row,
// `half` = which half of the features or keys) evaluate Phi_K, P and Phi_Q,
// stage the CTA's state, do the scan for the rows this CTA owns and run the
// epilogue; lane 0 of warp 8 issues the TMA loads and every tcgen05.mma;
// lane 0 of warp 9 publishes the state, gathers the scan's rows and loads
// the read-out operand.
#include <mutex>
#include <type_traits>

#include "../../include/taylor_attn.h"
#include "common.cuh"
#include "internal.h"
#include "phase.cuh"
#include "phi16.cuh"
#include "prefill_tc.h"
#include "ptx.cuh"
#include "tcgen05.cuh"
#include "tmap.h"

namespace ta {
namespace tc {

namespace {

using bf16 = __nv_bfloat16;

constexpr int kC = 128;        // tokens per chunk
constexpr int kDV = 64;
constexpr int kNV = 80;        // columns of [V | 1 | 0 ...]
constexpr int kFP = 160;       // features, padded
constexpr int kGroups = kFP / 8;
constexpr int kCompute = 256;
constexpr int kThreadsF = kCompute + 64;  // + the TMA / MMA warp (8) and the publishing warp (9)
constexpr int kMaxChunks = 36;  // chunks per head this kernel takes (the scan's gather fits the Phi_K space)
constexpr uint32_t kWaitPolls = 1u << 24;
constexpr uint32_t kFlagPolls = 1u << 24;

// shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kQBytes = kC * 16 * 2;           // 128 q (or k) rows, 32-byte swizzle
constexpr uint32_t kVAtom = 64 * 128;               // 64 v rows, 128-byte swizzle
constexpr uint32_t kOffQ = 0;                       // q of chunks a, b
constexpr uint32_t kOffK = kOffQ + 2 * kQBytes;     // k of chunks a, b
constexpr uint32_t kOffV = kOffK + 2 * kQBytes;     // four v atoms (two per chunk)
constexpr uint32_t kOffOnes = kOffV + 4 * kVAtom;   // the ones atom: column 64 of [V | 1 | 0]
constexpr uint32_t kOffPhi = kOffOnes + kVAtom;     // Phi_K hi, lo; then the scan's gather; then E of chunk b
constexpr uint32_t kPhiBytes = kC * 160 * 2;        // Phi_K hi (or lo)
constexpr uint32_t kGroupBytes = 8 * 2 * kNV * 2;   // one 8-feature group of E: [8][hi 80 | lo 80] bf16
constexpr uint32_t kEBytes = kGroups * kGroupBytes; // 51,200
constexpr int kXStride = 68;                        // published chunk state rows: [160][68] fp32
constexpr int kXFloats = kFP * kXStride;
constexpr uint32_t kRowBytes = kXStride * 4;        // one feature row of a published chunk state: 272
constexpr uint32_t kGatherMax = 320 * kRowBytes;    // the scan's gather: chunks x rows per owner <= 320
constexpr uint32_t kPhiSpace = 2 * kPhiBytes > kGatherMax ? 2 * kPhiBytes : kGatherMax;
constexpr uint32_t kOffE = kOffPhi + kPhiSpace;     // E of chunk a
constexpr uint32_t kSmemF = kOffE + kEBytes + 1024; // + alignment slack
constexpr uint32_t kLboPhi = (kFP / 8) * 128;       // K-group stride of Phi_K (MN-major)
constexpr uint32_t kOutTile = kC * 128;             // output staging: [128 rows][32 fp32], 128-byte swizzle
constexpr uint32_t kLboE = kGroupBytes;             // K-group stride of E (MN-major)
static_assert(kEBytes <= 2 * kPhiBytes, "E of chunk b fits the Phi_K space");
static_assert(4 * kOutTile <= kPhiSpace, "the output tiles of both chunks fit the Phi_K space");
static_assert(kSmemF <= 232448, "shared memory");

// TMEM (512 columns): the CTA's state T^T [0, 160); later the scores / P of
// the pairwise rounds, in two buffers [0, 128) and [160, 288) used in turn;
// later Phi_Q,a [0, 160) (hi 80 | lo 80) and Phi_Q,b [160, 320); O_a [320, 400),
// O_b [400, 480)
constexpr uint32_t kTT = 0, kTO = 320;
constexpr uint32_t kPBuf = 160;  // the second scores / P buffer (columns 160..287)

__device__ __forceinline__ bool waitb(uint64_t* bar, uint32_t parity, volatile int* bad) {
    return ptx::mbar_wait_or_abort(bar, parity, kWaitPolls, bad);
}

__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
    const uint32_t a = ptx::smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// named barrier of the 256 CUDA-core threads
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 1, %0;" ::"r"(kCompute) : "memory"); }

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Orders memory this thread has observed (through an acquire) before its
// later bulk copies, which read through the async proxy.
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Waits (one thread) until the counter reaches `target`; false, with *bad
// set, if the bound runs out or another role has failed.
__device__ bool wait_count(const unsigned* counter, unsigned target, volatile int* bad) {
    uint32_t it = 0;
    while (ld_acquire(counter) < target) {
        if (++it > kFlagPolls || *bad) {
            *bad = 1;
            return false;
        }
    }
    return true;
}

// One row of 16 bf16 from a 32-byte-swizzled K-major operand (as TMA writes
// it): 16-byte chunk c of row r sits at chunk c ^ ((r >> 2) & 1).
__device__ __forceinline__ void ld_row_sw32(const uint8_t* base, int r, float (&x)[16]) {
    const uint8_t* row = base + r * 32;
    const int sw = (r >> 2) & 1;
    const uint4 a = *reinterpret_cast<const uint4*>(row + ((0 ^ sw) << 4));
    const uint4 b = *reinterpret_cast<const uint4*>(row + ((1 ^ sw) << 4));
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// column 64 of [V | 1 | 0 ...] for 64 token rows under the 128-byte swizzle
__device__ __forceinline__ void init_ones(uint8_t* atom, int tid, int nthreads) {
    for (int i = tid; i < 64 * 8; i += nthreads) {
        const int k = i >> 3, c = i & 7;
        *reinterpret_cast<uint4*>(atom + k * 128 + ((c ^ (k & 7)) << 4)) = make_uint4(c == 0 ? 0x3F80u : 0u, 0, 0, 0);
    }
}

struct FusedArgs {
    const float* state_in;
    float* state_out;
    float* TG;        // [BH][NS][160][68] published states, one per CTA (its chunks together)
    uint8_t* EG;      // [BH][NS][kEBytes] read-out operands of the state before each CTA
    unsigned* flags;  // [BH] published chunk states, then [BH] finished feature groups (counters)
    int N, n, F, NC, NCH, ngroups, BH;
    float tau;
    int64_t stride;
    unsigned int* err;
};

__global__ void __launch_bounds__(kThreadsF, 1)
tc_fused_prefill_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                        const FusedArgs A) {
    extern __shared__ uint8_t sm_raw[];
    uint8_t* sm = align1k(sm_raw);
    __shared__ __align__(8) uint64_t ld, phik_full, phik_free, t_done, t_free, sc_full[2], p_full[2], p_free[2], gath,
        e_loaded[2], phiq_full[2], ro_done[2], t_staged;
    __shared__ uint32_t tslot;
    __shared__ int s_bad, s_e_issued[2], s_gath_issued, s_out_issued;
    volatile int* bad = &s_bad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int seg = blockIdx.x, bh = blockIdx.y;
    TA_PHASE(0, 0, tid == 0);
    const int n = A.n, F = A.F, NC = A.NC, NCH = A.NCH, ngroups = A.ngroups;
    const int c0 = seg * NCH;                                   // first chunk of this CTA
    const int nch = min(NCH, NC - c0);                          // its chunks (1 or 2)
    const int nrounds = nch == 2 ? 3 : 1;                       // pairwise blocks: aa (, bb, ba)
    const int64_t t0 = (int64_t)c0 * kC;
    const int rem = A.N - (int)t0;
    const int nval0 = min(kC, rem), nval1 = max(0, min(kC, rem - kC));  // valid rows of chunks a, b
    // chunk x reads out E_{c0 + x}, zero only for the head's first chunk without a carried state
    const bool inter0 = c0 > 0 || A.state_in != nullptr;
    const int NS = (NC + NCH - 1) / NCH;                        // CTAs of a head

    uint8_t* sQ = sm + kOffQ;
    uint8_t* sK = sm + kOffK;
    uint8_t* sV = sm + kOffV;
    uint8_t* sOnes = sm + kOffOnes;
    uint8_t* sPhi = sm + kOffPhi;  // Phi_K hi, lo; the scan's gather; E of chunk b
    uint8_t* sE = sm + kOffE;      // E of chunk a
    unsigned* tcount = A.flags + bh;          // chunk states of this head published
    unsigned* gcount = A.flags + A.BH + bh;   // feature groups of this head scanned

    if (tid == 0) {
        ptx::mbar_init(&ld, 1);
        ptx::mbar_init(&phik_full, kCompute);
        ptx::mbar_init(&phik_free, 1);
        ptx::mbar_init(&t_done, 1);
        ptx::mbar_init(&t_free, kCompute);
        for (int i = 0; i < 2; ++i) {  // one set per scores / P buffer
            ptx::mbar_init(&sc_full[i], 1);
            ptx::mbar_init(&p_full[i], kCompute);
            ptx::mbar_init(&p_free[i], 1);
        }
        ptx::mbar_init(&gath, 1);
        ptx::mbar_init(&t_staged, 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&e_loaded[i], 1);
            ptx::mbar_init(&phiq_full[i], kCompute);
            ptx::mbar_init(&ro_done[i], 1);
            s_e_issued[i] = 0;
        }
        s_bad = 0;
        s_gath_issued = 0;
        s_out_issued = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 8) {
        tmem_alloc(&tslot, 512);
        tmem_relinquish();
    }
    init_ones(sOnes, tid, kThreadsF);
    ptx::fence_proxy_async_smem();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tslot;

    if (warp == 8) {
        if (lane == 0) {
            // ------------------------------------------------ TMA loads and MMA issue
            ptx::mbar_arrive_expect_tx(&ld, (uint32_t)nch * (2 * kQBytes + 2 * kVAtom));
            for (int x = 0; x < nch; ++x) {
                const int y = (int)(t0 + x * kC);
                ptx::tma_load_3d(sQ + x * kQBytes, &tmq, 0, y, bh, &ld);
                ptx::tma_load_3d(sK + x * kQBytes, &tmk, 0, y, bh, &ld);
                ptx::tma_load_3d(sV + (2 * x) * kVAtom, &tmv, 0, y, bh, &ld);
                ptx::tma_load_3d(sV + (2 * x + 1) * kVAtom, &tmv, 0, y + 64, bh, &ld);
            }
            const uint32_t id_st = idesc_bf16(128, kFP, 1, 1);
            const uint32_t id80 = idesc_bf16(kC, kNV, 0, 1);
            // [V | 1 | 0] of chunk x, 16 token rows starting at row 16 ks
            // (MN-major, 128-byte swizzle; the ones atom through LBO)
            auto vdesc = [&](int x, int ks) -> uint64_t {
                const uint8_t* atom = sV + (2 * x + (ks >> 2)) * kVAtom;
                return smem_desc_sw(atom, (uint32_t)(sOnes - atom), 1024, kSwizzle128) + 128 * (ks & 3);
            };
            // the CTA's state: both chunks into one accumulator
            auto state = [&](int x) {
                const uint64_t ph = smem_desc(sPhi, kLboPhi, 128), pl = smem_desc(sPhi + kPhiBytes, kLboPhi, 128);
                const uint32_t d = tb + kTT;
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks) {
                    const uint64_t vd = vdesc(x, ks);
                    mma_bf16(d, vd, ph + (2 * kLboPhi / 16) * ks, id_st, (x > 0 || ks > 0) ? 1u : 0u);
                    mma_bf16(d, vd, pl + (2 * kLboPhi / 16) * ks, id_st, 1u);
                }
            };
            // round r: queries of chunk qx(r) against keys of chunk kx(r), in
            // scores / P buffer r % 2 (TMEM columns 0..127 or 160..287)
            auto qxr = [](int r) { return r == 0 ? 0 : 1; };
            auto kxr = [](int r) { return r == 1 ? 1 : 0; };
            auto scores = [&](int r) {
                const uint64_t qd = smem_desc_sw(sQ + qxr(r) * kQBytes, 16, 256, kSwizzle32);
                const uint64_t kd = smem_desc_sw(sK + kxr(r) * kQBytes, 16, 256, kSwizzle32);
                mma_bf16(tb + kTT + kPBuf * (r & 1), qd, kd, idesc_bf16(kC, kC, 0, 0), 0u);
                mma_commit(&sc_full[r & 1]);
            };
            // P of keys 16 ks .. 16 ks + 15: hi words at 32 (ks / 2) + 8 (ks % 2), lo 16 further
            auto pv = [&](int r) {
                const int ox = qxr(r), vx = kxr(r);
#pragma unroll
                for (int ks = 0; ks < kC / 16; ++ks) {
                    const uint32_t a = tb + kTT + kPBuf * (r & 1) + 32 * (ks >> 1) + 8 * (ks & 1);
                    const uint64_t vd = vdesc(vx, ks);
                    mma_bf16_ts(tb + kTO + 80 * ox, a, vd, id80, (r == 2 || ks > 0) ? 1u : 0u);
                    mma_bf16_ts(tb + kTO + 80 * ox, a + 16, vd, id80, 1u);
                }
                mma_commit(&p_free[r & 1]);
            };
            bool go = waitb(&ld, 0, bad);
            TA_PHASE(1, 1, true);
            // the chunk states (Phi_K of one chunk at a time in shared memory)
            for (int x = 0; x < nch && go; ++x) {
                go = waitb(&phik_full, x & 1, bad);
                if (go) {
                    fence_after_sync();
                    state(x);
                    mma_commit(x + 1 < nch ? &phik_free : &t_done);
                }
            }
            TA_PHASE(1, 2, true);
            // the pairwise parts, into the columns the state has left: round 0
            // chunk a against itself, round 1 chunk b against itself, round 2
            // chunk b against all of chunk a (which its read-out then leaves out)
            go = go && waitb(&t_free, 0, bad);
            if (go) {
                fence_after_sync();
                for (int r = 0; r < nrounds && r < 2; ++r) scores(r);
            }
            for (int r = 0; r < nrounds && go; ++r) {
                go = waitb(&p_full[r & 1], (r >> 1) & 1, bad);
                if (go) {
                    fence_after_sync();
                    pv(r);
                }
                if (go && r + 2 < nrounds) {  // its buffer again, once pv(r) has read P
                    go = waitb(&p_free[r & 1], (r >> 1) & 1, bad);
                    if (go) {
                        fence_after_sync();
                        scores(r + 2);
                    }
                }
            }
            TA_PHASE(1, 3, true);
            // the read-outs through the state before the CTA (one operand for both chunks)
            for (int x = 0; x < nch; ++x) {
                if (inter0) {
                    go = go && waitb(&phiq_full[x], 0, bad) && waitb(&e_loaded[0], 0, bad);
                    TA_PHASE(1, 10 + 2 * x, true);
                    if (go) {
                        fence_after_sync();
                        uint8_t* e = sE;
                        const uint64_t eh = smem_desc(e, kLboE, 128), el = smem_desc(e + 10 * 128, kLboE, 128);
                        const uint32_t dst = tb + kTO + 80 * x;
#pragma unroll
                        for (int ks = 0; ks < kFP / 16; ++ks) {
                            const uint32_t ah = tb + kTT + 160 * x + 8 * ks, al = ah + 80;
                            mma_bf16_ts(dst, ah, eh + (2 * kLboE / 16) * ks, id80, 1u);
                            mma_bf16_ts(dst, ah, el + (2 * kLboE / 16) * ks, id80, 1u);
                            mma_bf16_ts(dst, al, eh + (2 * kLboE / 16) * ks, id80, 1u);
                        }
                    }
                }
                mma_commit(&ro_done[x]);  // covers every MMA issued so far, also after a failure
                TA_PHASE(1, 11 + 2 * x, true);
            }
            TA_PHASE(1, 4, true);
            if (!go) *bad = 1;
        }
    } else if (warp == 9) {
        if (lane == 0) {
            // ------------------------------------------------ publishing the state
            // the staged T^T rows leave in one bulk store; once it has
            // completed, the head's count of published states grows
            if (waitb(&t_staged, 0, bad)) {
                ptx::bulk_s2g(A.TG + ((int64_t)bh * NS + seg) * kXFloats, sPhi, (uint32_t)kXFloats * 4u);
                ptx::bulk_commit();
                ptx::bulk_wait_all();
                fence_proxy_async_global();
                __threadfence();
                TA_PHASE(1, 9, true);
                if (!*bad) red_release_add(tcount, 1u);
                // the scan's gather: rows [R seg, R seg + nrows) of every state of
                // the head (the bulk store above has read the staging space)
                const int R = (F + NS - 1) / NS, f_lo = R * seg, nrows = max(0, min(R, F - f_lo));
                if (nrows > 0) {
                    if (!*bad && wait_count(tcount, (unsigned)NS, bad)) {
                        TA_PHASE(1, 5, true);
                        fence_proxy_async_global();
                        s_gath_issued = 1;
                        const uint32_t bytes = (uint32_t)nrows * kRowBytes;
                        ptx::mbar_arrive_expect_tx(&gath, (uint32_t)NS * bytes);
                        const float* src = A.TG + (int64_t)bh * NS * kXFloats + (int64_t)f_lo * kXStride;
                        for (int c = 0; c < NS; ++c)
                            ptx::bulk_g2s(sPhi + c * bytes, src + (int64_t)c * kXFloats, bytes, &gath);
                    } else {
                        atomicOr(A.err, kErrPrefillPipe);
                        *bad = 1;
                    }
                }
                // the read-out operand of the state before this CTA, once every
                // feature row of the head is scanned
                if (inter0) {
                    if (!*bad && wait_count(gcount, (unsigned)F, bad)) {
                        fence_proxy_async_global();
                        s_e_issued[0] = 1;
                        ptx::mbar_arrive_expect_tx(&e_loaded[0], (uint32_t)ngroups * kGroupBytes);
                        ptx::bulk_g2s(sE, A.EG + ((int64_t)bh * NS + seg) * kEBytes, (uint32_t)ngroups * kGroupBytes,
                                      &e_loaded[0]);
                    } else {
                        atomicOr(A.err, kErrPrefillPipe);
                        *bad = 1;
                    }
                }
            }
        }
    } else {
        // ---------------------------------------------------- CUDA-core roles
        const int row = (warp & 3) * 32 + lane, half = warp >> 2;
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        bool ok = waitb(&ld, 0, bad);
        TA_PHASE(0, 1, tid == 0);
        const float c1 = n >= 2 ? A.tau : 0.f, c2 = n >= 3 ? 0.5f * A.tau * A.tau : 0.f;

        // stage the CTA's state T^T (lane = v column, 160 feature columns) as
        // [feature][column] rows in the Phi_K space, which the state MMAs have
        // finished reading; the publishing warp takes them to L2
        auto stage_state = [&]() {
            ok = ok && waitb(&t_done, 0, bad);
            TA_PHASE(0, 3, tid == 0);
            if (ok) {
                fence_after_sync();
                if ((warp & 3) < 3) {
                    const int vc = row;  // lanes 0..64: v columns 0..63 and z
                    float* tg = reinterpret_cast<float*>(sPhi);
#pragma unroll
                    for (int p = 0; p < 5; ++p) {
                        float r[16];
                        tmem_ld16(tb + kTT + lane_off + 80 * half + 16 * p, r);
                        tmem_ld_wait();
                        if (vc <= kDV) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) tg[(80 * half + 16 * p + i) * kXStride + vc] = r[i];
                        }
                    }
                }
                fence_before_sync();
                ptx::mbar_arrive(&t_free);
                // E of chunk a: its groups past the last feature group stay zero
                for (uint32_t o = (uint32_t)ngroups * kGroupBytes + 16u * tid; o < kEBytes; o += 16u * kCompute)
                    *reinterpret_cast<uint4*>(sE + o) = make_uint4(0, 0, 0, 0);
            }
            // the staged rows go to the publishing warp's bulk store
            ptx::fence_proxy_async_smem();
            compute_sync();
            if (tid == 0 && ok && !*bad) ptx::mbar_arrive(&t_staged);
            TA_PHASE(0, 4, tid == 0);
        };

        // P = poly(tau q.k) of query `row` against keys [64 half, 64 half + 64),
        // each 32-key piece written in place over its own scores columns as
        // the TMEM A operand (16 hi words, then 16 lo words)
        auto p_rounds = [&](int r0, int r1) {
            for (int r = r0; r < r1 && ok; ++r) {
                ok = waitb(&sc_full[r & 1], (r >> 1) & 1, bad);
                if (!ok) break;
                fence_after_sync();
                const bool causal = r < 2;  // round 2: chunk b against all of chunk a
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const uint32_t tp = tb + kTT + kPBuf * (r & 1) + lane_off + 64 * half + 32 * pc;
                    float sc[32];
                    tmem_ld32(tp, sc);
                    tmem_ld_wait();
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float p2[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            float p = fmaf(fmaf(c2, sc[j + e], c1), sc[j + e], 1.f);
                            if (causal && 64 * half + 32 * pc + j + e > row) p = 0.f;
                            p2[e] = p;
                        }
                        split2(p2[0], p2[1], hi[j >> 1], lo[j >> 1]);
                    }
                    tmem_st16(tp, hi);
                    tmem_st16(tp + 16, lo);
                }
                tmem_st_wait();
                fence_before_sync();
                ptx::mbar_arrive(&p_full[r & 1]);
            }
        };

        // the scan: this CTA owns features [R seg, R seg + R) of its head (R =
        // ceil(F / NS)); it gathers those rows of every chunk state of the head
        // into shared memory, turns them in place into exclusive prefixes (one
        // thread per feature and column walks the chunks), then converts every
        // chunk's prefix into its rows of that chunk's hi/lo operand; the owner
        // of the last rows also writes the zero rows F .. 8 ngroups - 1
        auto scan = [&]() {
            const float* sin = A.state_in ? A.state_in + (int64_t)bh * A.stride : nullptr;
            float* gbuf = reinterpret_cast<float*>(sPhi);  // [NS][R][68]
            const int R = (F + NS - 1) / NS;
            const int f_lo = R * seg, nrows = max(0, min(R, F - f_lo));
            if (nrows == 0) return;
            // the publishing warp gathers this CTA's rows of every state of
            // the head into the Phi_K space once all of them are published
            const bool have = ok && !*bad && waitb(&gath, 0, bad);
            TA_PHASE(1, 6, tid == 0);
            const int cstride = nrows * kXStride;  // floats per chunk in the gather
            if (have) {
                for (int e = tid; e < nrows * (kDV + 1); e += kCompute) {
                    const int fr = e / (kDV + 1), col = e % (kDV + 1), f = f_lo + fr;
                    // plain loads: state_out may alias state_in (each element is
                    // read before it is written, by the same thread)
                    float run = 0.f;
                    if (sin) run = col < kDV ? sin[(int64_t)f * kDV + col] : sin[(int64_t)F * kDV + f];
                    float* gcol = gbuf + fr * kXStride + col;
                    for (int c = 0; c < NS; ++c) {
                        const float x = gcol[c * cstride];
                        gcol[c * cstride] = run;
                        run += x;
                    }
                    if (A.state_out) {
                        float* so = A.state_out + (int64_t)bh * A.stride;
                        if (col < kDV) so[(int64_t)f * kDV + col] = run;
                        else so[(int64_t)F * kDV + f] = run;
                    }
                }
            }
            compute_sync();
            TA_PHASE(1, 7, tid == 0);
            if (have) {
                // chunk c, column piece c8 (8 columns), feature row fr: 16 bytes hi, 16 lo
                const int erows = f_lo + nrows == F ? 8 * ngroups - f_lo : nrows;
                const int per_chunk = erows * 10;
                uint8_t* ebase = A.EG + (int64_t)bh * NS * kEBytes;
                for (int u = tid; u < NS * per_chunk; u += kCompute) {
                    const int c = u / per_chunk, r = u % per_chunk, c8 = r / erows, fr = r % erows, f = f_lo + fr;
                    const float* xr = gbuf + c * cstride + fr * kXStride + 8 * c8;
                    float x8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (fr >= nrows) {
                        // padding row: stays zero
                    } else if (c8 < 8) {
                        const float4 a0 = reinterpret_cast<const float4*>(xr)[0];
                        const float4 a1 = reinterpret_cast<const float4*>(xr)[1];
                        x8[0] = a0.x; x8[1] = a0.y; x8[2] = a0.z; x8[3] = a0.w;
                        x8[4] = a1.x; x8[5] = a1.y; x8[6] = a1.z; x8[7] = a1.w;
                    } else if (c8 == 8) {
                        x8[0] = xr[0];  // z; columns 65..79 stay zero
                    }
                    uint4 hi, lo;
                    split8(x8, hi, lo);
                    uint8_t* d = ebase + (int64_t)c * kEBytes + (f >> 3) * kGroupBytes + c8 * 128 + (f & 7) * 16;
                    *reinterpret_cast<uint4*>(d) = hi;
                    *reinterpret_cast<uint4*>(d + 10 * 128) = lo;
                }
            }
            TA_PHASE(1, 8, tid == 0);
            // every thread's rows, then one release at GPU scope (cumulative
            // over the CTA barrier) for the head's count of scanned rows
            compute_sync();
            if (tid == 0 && !*bad) red_release_add(gcount, (unsigned)nrows);
        };

        // Feature rows, one code path for both sides, so that the query side
        // runs on instructions the key side has already fetched: when the
        // kernel's code is in no cache, L2 included (as after other work has
        // streamed through L2), the first pass through this straight-line
        // code takes several times as long as later ones.  Code laid out right
        // after a wait is fetched during it, so the other phases follow the
        // key side in the loop body, in the order they run.  Pass j < 2 writes
        // Phi_K of chunk j, token `row`, features [80 half, 80 half + 80), hi
        // and lo, into the MN-major shared-memory operand; pass j >= 2 writes
        // c (.) Phi_Q of chunk j - 2 into TMEM (half 0 features 0..79 = words
        // 0..39 of the hi and lo halves, half 1 features 80..159).  Between the
        // two sides (after the second key-side pass): the staged state, the
        // pairwise rounds and the scan.
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
            const bool qside = j >= 2;
            const int x = j & 1;
            bool active = ok && x < nch && (!qside || inter0);
            if (active && j == 1) active = ok = waitb(&phik_free, 0, bad);
            if (active) {
                fence_after_sync();
                float x16[16];
                ld_row_sw32((qside ? sQ : sK) + x * kQBytes, row, x16);
                const bool valid = row < (x == 0 ? nval0 : nval1);
                const float e0 = valid ? 1.f : 0.f;
                const float e1 = qside ? c1 : ((valid && n >= 2) ? 1.f : 0.f);
                const float e2 = qside ? c2 : ((valid && n >= 3) ? 1.f : 0.f);
                // all 80 features of this half first (hi and lo words in registers),
                // then one store sequence per side
                uint32_t hw[40], lw[40];
                auto eval = [&](auto fb) {
                    constexpr int F0 = decltype(fb)::value;
                    constexpr int W = (F0 % 80) / 2;
                    float o[16];
                    phi16_range<F0, F0 + 16>(x16, e0, e1, e2, o);
#pragma unroll
                    for (int i = 0; i < 8; ++i) split2(o[2 * i], o[2 * i + 1], hw[W + i], lw[W + i]);
                };
                if (half == 0) {
                    eval(std::integral_constant<int, 0>());
                    eval(std::integral_constant<int, 16>());
                    eval(std::integral_constant<int, 32>());
                    eval(std::integral_constant<int, 48>());
                    eval(std::integral_constant<int, 64>());
                } else {
                    eval(std::integral_constant<int, 80>());
                    eval(std::integral_constant<int, 96>());
                    eval(std::integral_constant<int, 112>());
                    eval(std::integral_constant<int, 128>());
                    eval(std::integral_constant<int, 144>());
                }
                if (qside) {
                    // words 40 half .. 40 half + 39 of the hi and lo TMEM rows
                    const uint32_t th = tb + kTT + 160 * x + lane_off + 40 * half, tl = th + 80;
                    tmem_st32(th, *reinterpret_cast<const uint32_t(*)[32]>(hw));
                    tmem_st8(th + 32, *reinterpret_cast<const uint32_t(*)[8]>(hw + 32));
                    tmem_st32(tl, *reinterpret_cast<const uint32_t(*)[32]>(lw));
                    tmem_st8(tl + 32, *reinterpret_cast<const uint32_t(*)[8]>(lw + 32));
                } else {
                    // groups 10 half .. 10 half + 9 of the MN-major operand
#pragma unroll
                    for (int g = 0; g < 10; ++g) {
                        const uint32_t off = mnmaj(row, 10 * half + g, kLboPhi);
                        *reinterpret_cast<uint4*>(sPhi + off) =
                            make_uint4(hw[4 * g], hw[4 * g + 1], hw[4 * g + 2], hw[4 * g + 3]);
                        *reinterpret_cast<uint4*>(sPhi + kPhiBytes + off) =
                            make_uint4(lw[4 * g], lw[4 * g + 1], lw[4 * g + 2], lw[4 * g + 3]);
                    }
                }
                if (qside) {
                    tmem_st_wait();
                    ptx::fence_proxy_async_smem();  // the zeroed tails of E
                    fence_before_sync();
                    ptx::mbar_arrive(&phiq_full[x]);
                    TA_PHASE(0, 11 + x, tid == 0);
                } else {
                    ptx::fence_proxy_async_smem();
                    ptx::mbar_arrive(&phik_full);
                }
            }
            if (j == 1) {
                TA_PHASE(0, 2, tid == 0);
                stage_state();
                // every round now, while the states are published and gathered
                p_rounds(0, nrounds);
                TA_PHASE(0, 5, tid == 0);
                scan();
                if (A.state_out && seg == 0)
                    for (int64_t e = (int64_t)F * (kDV + 1) + tid; e < A.stride; e += kCompute)
                        A.state_out[(int64_t)bh * A.stride + e] = 0.f;
                TA_PHASE(0, 6, tid == 0);
                // c (.) Phi_Q goes where the scores / P buffers were: every P
                // consumed (buffer 0 was used (nrounds + 1) / 2 times, buffer 1
                // nrounds / 2)
                if (inter0) {
                    TA_PHASE(0, 7, tid == 0);
                    ok = ok && waitb(&p_free[0], (((nrounds + 1) >> 1) - 1) & 1, bad);
                    if (nrounds > 1) ok = ok && waitb(&p_free[1], ((nrounds >> 1) - 1) & 1, bad);
                }
            }
        }
        TA_PHASE(0, 8, tid == 0);

        // epilogues: o = numerator * (1 / denominator), staged as two
        // [128 rows][32 columns] fp32 tiles a chunk under the 128-byte swizzle
        // (in the Phi_K space, idle since the scan) and written by TMA tensor
        // stores, which leave out the rows past the sequence.  Per-thread
        // global stores would fill the SM's memory pipeline while the other
        // chunk's read-out is still being issued.
        for (int x = 0; x < nch; ++x) {
            const bool done = waitb(&ro_done[x], 0, bad);
            fence_after_sync();
            TA_PHASE(0, 13 + x, tid == 0);
            if (done && !*bad) {
                float o[32];
                const uint32_t to = tb + kTO + 80 * x + lane_off;
                tmem_ld32(to + 32 * half, o);
                const float dn = tmem_ld1(to + kDV);
                tmem_ld_wait();
                const float rcp = __frcp_rn(dn);
                uint8_t* trow = sPhi + (2 * x + half) * kOutTile + row * 128;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    *reinterpret_cast<float4*>(trow + ((i ^ (row & 7)) << 4)) =
                        make_float4(o[4 * i] * rcp, o[4 * i + 1] * rcp, o[4 * i + 2] * rcp, o[4 * i + 3] * rcp);
            }
            ptx::fence_proxy_async_smem();
            compute_sync();
            if (tid == 0 && !*bad) {
                const int y = (int)(t0 + x * kC);
                ptx::tma_store_3d(&tmo, 0, y, bh, sPhi + (2 * x) * kOutTile);
                ptx::tma_store_3d(&tmo, 32, y, bh, sPhi + (2 * x + 1) * kOutTile);
                ptx::bulk_commit();
                s_out_issued = 1;
            }
        }
        TA_PHASE(0, 9, tid == 0);
    }

    // every copy and MMA this CTA started has landed before it leaves
    __syncthreads();
    TA_PHASE(0, 10, tid == 0);
    if (tid == 0) {
        if (!ptx::mbar_wait(&ld, 0, kWaitPolls)) s_bad = 1;
        if (!ptx::mbar_wait(&ro_done[nch - 1], 0, kWaitPolls)) s_bad = 1;
        for (int x = 0; x < 2; ++x)
            if (s_e_issued[x] && !ptx::mbar_wait(&e_loaded[x], 0, kWaitPolls)) s_bad = 1;
        // the last gather (each earlier one completed before the next was issued)
        if (s_gath_issued && !ptx::mbar_wait(&gath, 0, kWaitPolls)) s_bad = 1;
        // the output stores this thread issued
        if (s_out_issued) ptx::bulk_wait_all();
        if (s_bad) atomicOr(A.err, kErrPrefillPipe);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 8) {
        fence_after_sync();
        tmem_dealloc(tb, 512);
    }
}

constexpr int kMaxDevices = 64;

struct FusedSetup {
    cudaError_t attr = cudaErrorUnknown;
    int capacity = 0;  // CTAs that can be resident together
    int per_sm = 0;
};

FusedSetup setup_for_device(int dev) {
    static std::once_flag once[kMaxDevices];
    static FusedSetup res[kMaxDevices];
    std::call_once(once[dev], [dev]() {
        FusedSetup r;
        const void* fn = reinterpret_cast<const void*>(tc_fused_prefill_kernel);
        r.attr = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemF);
        int per_sm = 0, sms = 0, coop = 0;
        if (r.attr == cudaSuccess)
            r.attr = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, tc_fused_prefill_kernel, kThreadsF, kSmemF);
        if (r.attr == cudaSuccess) r.attr = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (r.attr == cudaSuccess) r.attr = cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
        if (r.attr != cudaSuccess) cudaGetLastError();
        // one CTA per SM: it allocates all of the SM's TMEM
        r.capacity = (coop && per_sm >= 1) ? sms : 0;
        r.per_sm = per_sm;
        res[dev] = r;
    });
    return res[dev];
}

}  // namespace

int try_prefill_fused(const __nv_bfloat16* q, const __nv_bfloat16* k, const __nv_bfloat16* v, float* out,
                      const float* state_in, float* state_out, int BH, int N, int d, int dv, int n, float tau,
                      int64_t F, int64_t stride, cudaStream_t stream) {
    if (d != 16 || dv != kDV || n > 3 || N <= 0 || BH <= 0 || BH > 65535) return kNotApplicable;
    const int NC = (N + kC - 1) / kC;
    if (NC > kMaxChunks) return kNotApplicable;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return kNotApplicable;
    }
    const FusedSetup su = setup_for_device(dev);
    if (su.attr != cudaSuccess || su.capacity == 0) return kNotApplicable;
    // one chunk per CTA when every chunk can have its own resident CTA, else two
    int NCH = 1;
    if ((int64_t)BH * NC > su.capacity) NCH = 2;
    const int NS = (NC + NCH - 1) / NCH;
    if ((int64_t)BH * NS > su.capacity) return kNotApplicable;
    // each CTA's share of the scan: R feature rows of every chunk state of its head
    const int R = (int)((F + NS - 1) / NS);
    if ((int64_t)NS * R * kRowBytes > kGatherMax) return kNotApplicable;
    unsigned int* err = device_error_word();
    if (!err) return TAYLOR_ERR_CUDA;

    CUtensorMap tmq, tmk, tmv, tmo;
    if (make_tmap_bf16_3d(&tmq, q, 16, (uint64_t)N, (uint64_t)BH, 16, kC, 32) != cudaSuccess ||
        make_tmap_bf16_3d(&tmk, k, 16, (uint64_t)N, (uint64_t)BH, 16, kC, 32) != cudaSuccess ||
        make_tmap_bf16_3d(&tmv, v, kDV, (uint64_t)N, (uint64_t)BH, kDV, 64, 128) != cudaSuccess ||
        make_tmap_f32_3d(&tmo, out, kDV, (uint64_t)N, (uint64_t)BH, (uint64_t)kDV * 4, (uint64_t)N * kDV * 4, 32, kC,
                         128) != cudaSuccess)
        return kNotApplicable;

    // workspace: published chunk states, read-out operands, flags
    const int ngroups = (int)((F + 7) / 8);
    const size_t tg_bytes = (size_t)BH * NS * kXFloats * sizeof(float);  // one state per CTA
    const size_t eg_bytes = (size_t)BH * NS * kEBytes;                    // one read-out operand per CTA
    const size_t fl_bytes = (size_t)2 * BH * sizeof(unsigned);
    uint8_t* ws = nullptr;
    if (workspace_alloc(reinterpret_cast<void**>(&ws), tg_bytes + eg_bytes + fl_bytes, stream) != cudaSuccess) {
        cudaGetLastError();
        return TAYLOR_ERR_OUT_OF_MEMORY;
    }
    FusedArgs a;
    a.state_in = state_in;
    a.state_out = state_out;
    a.TG = reinterpret_cast<float*>(ws);
    a.EG = ws + tg_bytes;
    a.flags = reinterpret_cast<unsigned*>(ws + tg_bytes + eg_bytes);
    a.N = N;
    a.n = n;
    a.F = (int)F;
    a.NC = NC;
    a.NCH = NCH;
    a.ngroups = ngroups;
    a.BH = BH;
    a.tau = tau;
    a.stride = stride;
    a.err = err;
    cudaError_t e = cudaMemsetAsync(a.flags, 0, fl_bytes, stream);
    if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(NS, BH, 1);
        cfg.blockDim = dim3(kThreadsF);
        cfg.dynamicSmemBytes = kSmemF;
        cfg.stream = stream;
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeCooperative;
        at[0].val.cooperative = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        TA_TIMED(stream, "tc_fused_prefill_kernel", e = cudaLaunchKernelEx(&cfg, tc_fused_prefill_kernel, tmq, tmk, tmv, tmo, a));
    }
    const cudaError_t e2 = workspace_free(ws, stream);
    if (e == cudaSuccess) e = e2;
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e == cudaErrorMemoryAllocation ? TAYLOR_ERR_OUT_OF_MEMORY : TAYLOR_ERR_CUDA;
    }
    return TAYLOR_OK;
}

}  // namespace tc
}  // namespace ta
