// Evaluation of 32 consecutive packed features of one token inside the
// tensor-core kernels, from the token's bf16 row held in shared memory as a
// row of a swizzled K-major operand: 16-byte chunk c of the row (elements
// 8c .. 8c+7) at rowbase + 16 (c ^ sw).
//
// Feature f (degree m, indices i1 <= ... <= im, weight sqrt(m!/alpha!); the
// packing of arXiv 2610.20637, abstract) is w * x_i1 * ... * x_im, times the
// query factor tau^m/m! on the query side.
//
// For the head sizes and orders the kernels specialise on, a block of 32
// features is unrolled at compile time: every index and weight is a
// constant, x stays in registers, only the 16-byte chunks of x that the block
// uses are loaded, and the products are written left to right so that the
// features of one run (same leading indices, last index increasing) share
// the prefix product; most features then cost one multiplication.  Other
// shapes take the run-time path, which reads per-feature descriptors.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"
#include "feature_table.cuh"

namespace ta {
namespace fe {

// ------------------------------------------------------------ compile-time tables
template <int D>
struct CtMax;
template <>
struct CtMax<16> {
    static constexpr int kN = 5;
};
template <>
struct CtMax<32> {
    static constexpr int kN = 4;
};
template <>
struct CtMax<64> {
    static constexpr int kN = 3;
};

template <int D>
inline constexpr FeatTable<D, CtMax<D>::kN> kCtTable = make_feat_table<D, CtMax<D>::kN>();

template <int D>
__host__ __device__ constexpr uint32_t ct_code(int f) {
    return kCtTable<D>.e[f].code;
}
template <int D>
__host__ __device__ constexpr float ct_weight(int f) {
    return kCtTable<D>.e[f].w;
}

// Bit c set when a feature of block b (features 32b .. 32b+31, those < nf)
// reads x from 16-byte chunk c (indices 8c .. 8c+7).
template <int D>
__host__ __device__ constexpr uint32_t ct_chunk_mask(int nf, int b) {
    uint32_t mask = 0;
    for (int f = 32 * b; f < 32 * b + 32 && f < nf; ++f) {
        const uint32_t code = ct_code<D>(f);
        const int m = (int)(code >> 24);
        for (int s = 0; s < m; ++s) mask |= 1u << (((code >> (6 * s)) & 63u) / 8);
    }
    return mask;
}

// x_i from the loaded chunks (bf16 -> fp32 is a shift).
template <int I, int NC>
__device__ __forceinline__ float xv(const uint4 (&ch)[NC]) {
    constexpr int c = I / 8, e = I % 8;
    uint32_t word;
    if constexpr (e / 2 == 0) word = ch[c].x;
    else if constexpr (e / 2 == 1) word = ch[c].y;
    else if constexpr (e / 2 == 2) word = ch[c].z;
    else word = ch[c].w;
    return __uint_as_float((e & 1) ? (word & 0xffff0000u) : (word << 16));
}

template <int D, int N, bool kQuery, int F>
__device__ __forceinline__ float ct_feature(const uint4 (&ch)[D / 8], const float (&qc)[N]) {
    if constexpr (F >= cx_num_features(D, N)) {
        return 0.f;
    } else {
        constexpr uint32_t code = ct_code<D>(F);
        constexpr int m = (int)(code >> 24);
        constexpr float w = ct_weight<D>(F);
        float c;
        if constexpr (kQuery) c = qc[m] * w;
        else c = w;
        if constexpr (m >= 1) c = c * xv<(int)(code & 63u)>(ch);
        if constexpr (m >= 2) c = c * xv<(int)((code >> 6) & 63u)>(ch);
        if constexpr (m >= 3) c = c * xv<(int)((code >> 12) & 63u)>(ch);
        if constexpr (m >= 4) c = c * xv<(int)((code >> 18) & 63u)>(ch);
        return c;
    }
}

template <uint32_t kMask, int C, int NC>
__device__ __forceinline__ void ct_load_chunk(const uint8_t* rowbase, uint32_t sw, uint4 (&ch)[NC]) {
    if constexpr ((kMask >> C) & 1u) ch[C] = *reinterpret_cast<const uint4*>(rowbase + ((C ^ sw) << 4));
}

template <uint32_t kMask, int NC, int... C>
__device__ __forceinline__ void ct_load_chunks(const uint8_t* rowbase, uint32_t sw, uint4 (&ch)[NC],
                                               std::integer_sequence<int, C...>) {
    (ct_load_chunk<kMask, C>(rowbase, sw, ch), ...);
}

template <int D, int N, bool kQuery, int F0, int... E>
__device__ __forceinline__ void ct_fill(const uint4 (&ch)[D / 8], const float (&qc)[N], float (&o)[32],
                                        std::integer_sequence<int, E...>) {
    ((o[E] = ct_feature<D, N, kQuery, F0 + E>(ch, qc)), ...);
}

template <int D, int N, bool kQuery, int B>
__device__ __forceinline__ void ct_block(const uint8_t* rowbase, uint32_t sw, const float (&qc)[N], float (&o)[32]) {
    constexpr uint32_t kMask = ct_chunk_mask<D>(cx_num_features(D, N), B);
    uint4 ch[D / 8];
#pragma unroll
    for (int c = 0; c < D / 8; ++c) ch[c] = make_uint4(0, 0, 0, 0);
    ct_load_chunks<kMask>(rowbase, sw, ch, std::make_integer_sequence<int, D / 8>{});
    ct_fill<D, N, kQuery, 32 * B>(ch, qc, o, std::make_integer_sequence<int, 32>{});
}

// Binary dispatch on the run-time block index.
template <int D, int N, bool kQuery, int LO, int HI>
__device__ __forceinline__ void ct_dispatch(int b, const uint8_t* rowbase, uint32_t sw, const float (&qc)[N],
                                            float (&o)[32]) {
    if constexpr (HI - LO == 1) {
        ct_block<D, N, kQuery, LO>(rowbase, sw, qc, o);
    } else {
        constexpr int MID = (LO + HI) / 2;
        if (b < MID) ct_dispatch<D, N, kQuery, LO, MID>(b, rowbase, sw, qc, o);
        else ct_dispatch<D, N, kQuery, MID, HI>(b, rowbase, sw, qc, o);
    }
}

// ------------------------------------------------------------ run-time path
__device__ __forceinline__ float rt_x(const uint8_t* rowbase, uint32_t sw, int i) {
    const uint16_t h = *reinterpret_cast<const uint16_t*>(rowbase + ((((uint32_t)i >> 3) ^ sw) << 4) + (i & 7) * 2);
    return __uint_as_float((uint32_t)h << 16);
}

template <int D, bool kQuery>
__device__ __forceinline__ void rt_block(int b, const uint8_t* rowbase, uint32_t sw, const float* qc, int n, int F,
                                         float tau, float (&o)[32]) {
    const PackedFeat* tab = feat_table(D, n);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const int f = 32 * b + e;
        float c = 0.f;
        if (f < F) {
            const FeatDesc fd = get_desc(tab, D, n, f, tau, qc, kQuery);
            c = fd.w;
            for (int s = 0; s < fd.m; ++s) c *= rt_x(rowbase, sw, (fd.packed >> (8 * s)) & 0xff);
        }
        o[e] = c;
    }
}

// ------------------------------------------------------------ entry
// Features 32b .. 32b+31 of the token at rowbase.  N > 0: compile-time
// shape (D, N); N == 0: run-time order n (F features).  qc[m] = tau^m/m!
// (read on the query side only).
template <int D, int N, bool kQuery>
struct Eval {
    static constexpr bool kCompileTime = N > 0;
    __device__ static __forceinline__ void block(int b, const uint8_t* rowbase, uint32_t sw, const float* qc, int n,
                                                 int F, float tau, float (&o)[32]) {
        if constexpr (N > 0) {
            constexpr int kBlocks = (cx_num_features(D, N) + 31) / 32;
            if (b >= kBlocks) {  // a tile's blocks past the last feature
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = 0.f;
                return;
            }
            float q[N];
#pragma unroll
            for (int m = 0; m < N; ++m) q[m] = kQuery ? qc[m] : 1.f;
            ct_dispatch<D, N, kQuery, 0, kBlocks>(b, rowbase, sw, q, o);
        } else {
            rt_block<D, kQuery>(b, rowbase, sw, qc, n, F, tau, o);
        }
    }
};

}  // namespace fe
}  // namespace ta
