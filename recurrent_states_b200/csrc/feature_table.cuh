// Compile-time feature tables for the head sizes the kernels specialise on.
//
// A packed feature (arXiv 2610.20637, abstract: the m-th state is
// binom(d+m-1, m) wide) is a degree m <= 4 and indices i1 <= ... <= im < 64.
// The table for head size D lists every feature of degree < NMAX in the
// library's order (degree-major, lexicographic inside a degree).  Because the
// order is degree-major, the first F(D, n) entries of the table are exactly
// the features for any n <= NMAX.  Each entry is
//   code = i1 | i2 << 6 | i3 << 12 | i4 << 18 | m << 24,   w = sqrt(m!/alpha!)
// built by constexpr enumeration (the square root by Newton's iteration in
// double, which for these small integers lands on the correctly rounded float).
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace ta {

struct PackedFeat {
    uint32_t code;
    float w;
};

constexpr int64_t cx_binom(int a, int b) {
    if (b < 0 || a < 0 || b > a) return 0;
    int64_t r = 1;
    for (int i = 1; i <= b; ++i) r = r * (a - b + i) / i;
    return r;
}

constexpr int cx_num_features(int d, int n) {
    int64_t F = 0;
    for (int m = 0; m < n; ++m) F += cx_binom(d + m - 1, m);
    return (int)F;
}

constexpr double cx_sqrt(double x) {
    double r = x > 1.0 ? x : 1.0;
    for (int i = 0; i < 64; ++i) r = 0.5 * (r + x / r);
    return r;
}

template <int D, int NMAX>
struct FeatTable {
    static constexpr int F = cx_num_features(D, NMAX);
    PackedFeat e[F];
};

template <int D, int NMAX>
constexpr FeatTable<D, NMAX> make_feat_table() {
    FeatTable<D, NMAX> t{};
    int f = 0;
    for (int m = 0; m < NMAX; ++m) {
        int idx[4] = {0, 0, 0, 0};
        for (;;) {
            uint32_t code = (uint32_t)m << 24;
            for (int p = 0; p < m; ++p) code |= (uint32_t)idx[p] << (6 * p);
            int mf = 1;
            for (int s = 2; s <= m; ++s) mf *= s;
            int den = 1, run = 1;
            for (int p = 1; p <= m; ++p) {
                if (p < m && idx[p] == idx[p - 1]) {
                    ++run;
                } else {
                    for (int s = 2; s <= run; ++s) den *= s;
                    run = 1;
                }
            }
            t.e[f].code = code;
            t.e[f].w = (float)cx_sqrt((double)mf / (double)den);
            ++f;
            int p = m - 1;
            while (p >= 0 && idx[p] == D - 1) --p;
            if (p < 0) break;
            idx[p] += 1;
            for (int r = p + 1; r < m; ++r) idx[r] = idx[p];
        }
    }
    return t;
}

// Tables held in device memory (static, part of the library image; each
// translation unit that reads them carries its own copy).
static __device__ const FeatTable<16, 5> kFeat16 = make_feat_table<16, 5>();  // 4845: d_k 16, n <= 5
static __device__ const FeatTable<32, 4> kFeat32 = make_feat_table<32, 4>();  // 6545: d_k 32, n <= 4
static __device__ const FeatTable<64, 3> kFeat64 = make_feat_table<64, 3>();  // 2145: d_k 64, n <= 3

// Device pointer to the table that covers (d, n), or nullptr.
__device__ __forceinline__ const PackedFeat* feat_table(int d, int n) {
    if (d == 16 && n <= 5) return kFeat16.e;
    if (d == 32 && n <= 4) return kFeat32.e;
    if (d == 64 && n <= 3) return kFeat64.e;
    return nullptr;
}

__device__ __forceinline__ FeatDesc desc_from_packed(PackedFeat p, const float* qcoef, bool query) {
    FeatDesc fd;
    fd.m = (int)(p.code >> 24);
    fd.packed = 0;
    for (int s = 0; s < fd.m; ++s) fd.packed |= ((p.code >> (6 * s)) & 63u) << (8 * s);
    fd.w = query ? p.w * qcoef[fd.m] : p.w;
    return fd;
}

// Descriptor of feature f: from the static table when one covers (d, n),
// else by unranking.  qcoef[m] = tau^m/m! (used when query is true).
__device__ __forceinline__ FeatDesc get_desc(const PackedFeat* tab, int d, int n, int64_t f, float tau,
                                             const float* qcoef, bool query) {
    if (tab) return desc_from_packed(tab[f], qcoef, query);
    return make_desc(d, n, f, tau, query);
}

}  // namespace ta
