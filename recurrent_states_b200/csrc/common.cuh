// Shared device/host helpers of libtaylor_attn: the packed feature order
// (unranking a feature number into its monomial), the multinomial weights,
// and small load helpers.
//
// Packing (arXiv 2610.20637, abstract: each Taylor term factors into a
// tensor-power inner product and the m-th state is binom(d+m-1, m) wide):
// feature f is a degree m and indices i1 <= ... <= im; degrees are stored in
// increasing order and, inside a degree, the tuples in lexicographic order.
// phi_f(x) = sqrt(m!/alpha!) * x_{i1} * ... * x_{im}, alpha the multiplicities,
// so that sum over one degree of phi_f(q) phi_f(k) = (q.k)^m exactly.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define TA_HD __host__ __device__ __forceinline__

namespace ta {

constexpr int kMaxN = 5;      // terms of the series (degrees 0..4)
constexpr int kMaxDk = 64;
constexpr int kMaxDv = 256;

TA_HD int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// binom(a, b) for the library's range (a <= 68, b <= 4): 32-bit arithmetic
// suffices (largest intermediate 814385 * 68).
TA_HD int64_t binom(int a, int b) {
    if (b < 0 || a < 0 || b > a) return 0;
    int r = 1;
    for (int i = 1; i <= b; ++i) r = r * (a - b + i) / i;
    return r;
}

TA_HD int64_t num_features(int d, int n) {
    int64_t F = 0;
    for (int m = 0; m < n; ++m) F += binom(d + m - 1, m);
    return F;
}

// Monomial of feature f: degree m and indices idx[0..m-1] (non-decreasing).
struct Mono {
    int m;
    int idx[kMaxN - 1];
};

// Unrank f in the degree-major, lexicographic order.  The number of
// non-decreasing tuples of length r over the values [a, d) is
// binom(d - a + r - 1, r), which lets the loop skip whole subtrees.
TA_HD Mono unrank(int d, int n, int64_t f) {
    Mono mo;
    mo.m = 0;
    int64_t off = 0;
    while (mo.m < n - 1) {
        const int64_t w = binom(d + mo.m - 1, mo.m);
        if (f < off + w) break;
        off += w;
        ++mo.m;
    }
    int64_t r = f - off;
    int lo = 0;
    for (int p = 0; p < kMaxN - 1; ++p) mo.idx[p] = -1;
    for (int p = 0; p < mo.m; ++p) {
        const int rest = mo.m - p - 1;
        for (int a = lo; a < d; ++a) {
            const int64_t cnt = binom(d - a + rest - 1, rest);
            if (r < cnt) {
                mo.idx[p] = a;
                lo = a;
                break;
            }
            r -= cnt;
        }
    }
    return mo;
}

// sqrt(m! / alpha!) for a sorted index tuple.
TA_HD float mono_weight(const Mono& mo) {
    int mf = 1;
    for (int s = 2; s <= mo.m; ++s) mf *= s;
    int den = 1, run = 1;
    for (int p = 1; p <= mo.m; ++p) {
        if (p < mo.m && mo.idx[p] == mo.idx[p - 1]) {
            ++run;
        } else {
            for (int s = 2; s <= run; ++s) den *= s;
            run = 1;
        }
    }
    return sqrtf((float)mf / (float)den);
}

// tau^m / m!, the per-degree factor carried on the query side.
TA_HD float query_coeff(int m, float tau) {
    float c = 1.0f;
    for (int s = 1; s <= m; ++s) c = c * tau / (float)s;
    return c;
}

// Compact per-feature descriptor used by the kernels: up to four 8-bit
// indices packed in one word, the degree, and the weight (times the query
// factor when the feature is used on the query side).
struct FeatDesc {
    uint32_t packed;  // idx[p] in bits 8p..8p+7
    int m;
    float w;
};

TA_HD FeatDesc make_desc(int d, int n, int64_t f, float tau, bool query) {
    const Mono mo = unrank(d, n, f);
    FeatDesc fd;
    fd.m = mo.m;
    fd.packed = 0;
    for (int p = 0; p < mo.m; ++p) fd.packed |= (uint32_t)mo.idx[p] << (8 * p);
    fd.w = mono_weight(mo) * (query ? query_coeff(mo.m, tau) : 1.0f);
    return fd;
}

// Feature f of degree <= 2 over d_k = d, arithmetically (no table): degree m,
// indices i <= j and the multinomial weight sqrt(m!/alpha!) (sqrt 2 for
// i != j, else 1), in the order unrank() defines (degree-major, index pairs
// in lexicographic order).  Factors past the degree are to be taken as 1.
__device__ __forceinline__ void feature_deg2(int d, int f, int& m, int& i, int& j, float& w) {
    m = 0;
    i = 0;
    j = 0;
    w = 1.0f;
    if (f == 0) return;
    if (f <= d) {
        m = 1;
        i = f - 1;
        return;
    }
    int r = f - 1 - d, a = 0;
    while (r >= d - a) {
        r -= d - a;
        ++a;
    }
    m = 2;
    i = a;
    j = a + r;
    if (i != j) w = 1.41421356237309505f;
}

// phi_f(x) for x in shared memory with element stride 1.
__device__ __forceinline__ float eval_desc(const FeatDesc& fd, const float* x) {
    float p = fd.w;
    for (int s = 0; s < fd.m; ++s) p *= x[(fd.packed >> (8 * s)) & 0xff];
    return p;
}

template <typename T>
__device__ __forceinline__ float ldf(const T* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

// sum_{m<n} x^m/m! by Horner: 1 + x(1 + x/2(1 + x/3(...))).
__device__ __forceinline__ float taylor_kernel(float x, int n) {
    float w = 1.0f;
    for (int m = n - 1; m >= 1; --m) w = 1.0f + w * x / (float)m;
    return w;
}

}  // namespace ta
