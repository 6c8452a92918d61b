// Closed-form feature map for d_k = 16, n <= 3, shared by the tensor-core
// prefill kernels: phi = [1, x_i, w_ab x_a x_b (a <= b)] with w = sqrt(2) for
// a < b and 1 for a = b (the multinomial weights sqrt(m!/alpha!) of the
// packed order: degree-major, index pairs in lexicographic order), features
// 153..159 zero padding, each degree scaled by a caller factor (tau^m/m! on
// the query side, 1 on the key side, 0 for degrees >= n).
#pragma once

#include "tcgen05.cuh"

namespace ta {
namespace tc {

constexpr float kSqrt2 = 1.41421356237309504880f;
constexpr int kPhi16Width = 160;  // 153 features padded to a multiple of 16

// Writes features [8*G0, 8*G1) of the 160 padded features of one token,
// scaled per degree by (e0, e1, e2), as hi/lo bf16 groups of 8 through
// `put(group, hi, lo)`.  All indices are compile-time constants after
// unrolling, so features outside the range cost nothing.
template <int G0, int G1, typename Put>
__device__ __forceinline__ void phi16_groups(const float (&x)[16], float e0, float e1, float e2, Put put) {
    float buf[8];
    int f = 0;
    auto emit = [&](auto make) {
        if (f >= 8 * G0 && f < 8 * G1) {
            buf[f & 7] = make();
            if ((f & 7) == 7) {
                uint4 hi, lo;
                split8(buf, hi, lo);
                put(f >> 3, hi, lo);
            }
        }
        ++f;
    };
    emit([&] { return e0; });
#pragma unroll
    for (int i = 0; i < 16; ++i) emit([&] { return e1 * x[i]; });
    const float e2o = e2 * kSqrt2;
#pragma unroll
    for (int a = 0; a < 16; ++a) {
#pragma unroll
        for (int b = a; b < 16; ++b) emit([&] { return (a == b ? e2 : e2o) * x[a] * x[b]; });
    }
#pragma unroll
    for (int i = 153; i < kPhi16Width; ++i) emit([&] { return 0.f; });
}

// Features [F0, F1) of the same map into o[0 .. F1 - F0), each index a
// compile-time constant after unrolling (so o stays in registers):
// feature 0 is e0, 1 + i is e1 x_i, 17 + (16 a - a (a - 1) / 2) + (b - a) is
// the pair a <= b, 153..159 are zero.
template <int F0, int F1>
__device__ __forceinline__ void phi16_range(const float (&x)[16], float e0, float e1, float e2, float (&o)[F1 - F0]) {
    if (F0 == 0) o[0] = e0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int f = 1 + i;
        if (f >= F0 && f < F1) o[f - F0] = e1 * x[i];
    }
    const float e2o = e2 * kSqrt2;
#pragma unroll
    for (int a = 0; a < 16; ++a) {
#pragma unroll
        for (int b = a; b < 16; ++b) {
            const int f = 17 + 16 * a - a * (a - 1) / 2 + (b - a);
            if (f >= F0 && f < F1) o[f - F0] = (a == b ? e2 : e2o) * x[a] * x[b];
        }
    }
#pragma unroll
    for (int f = 153; f < kPhi16Width; ++f)
        if (f >= F0 && f < F1) o[f - F0] = 0.f;
}

}  // namespace tc
}  // namespace ta
