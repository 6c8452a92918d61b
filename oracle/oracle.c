/*
 * Float64 CPU oracle (plain C, OpenMP across heads) for causal attention with
 * a truncated-Taylor exponential kernel.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, by __graft_entry__.smoke() and
 * by the CPU-baseline / reference legs of bench.py.  It shares no code, table
 * or header with the CUDA library; it builds its own feature table.
 *
 * Source: "Expanding Attention: A Taylor-Series Route to Linear-Time
 * Transformers with a Fixed Number of Recurrent States" (arXiv 2610.20637),
 * abstract:
 *   - exp is cut after n Taylor terms: K(x) = sum_{m<n} x^m/m!, x = tau q.k;
 *   - each term is an inner product of tensor powers, packed to the
 *     binom(d+m-1, m) non-decreasing monomials with weight sqrt(m!/alpha!);
 *   - so the causal history is n states, S += phi(k) [v|1]^T per token.
 * Readings (not fixed by the paper's abstract): tau^m/m! on the query side, inclusive
 * causality, the ones column of [v|1] as normaliser, a plain quotient.
 *
 * Logical state layout here: S[head][F][dv+1] (last column = normaliser).
 * All functions return 0 on success, a negative value on a bad argument.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static long binom_l(long a, long b) {
    if (b < 0 || b > a) return 0;
    long r = 1;
    for (long i = 1; i <= b; ++i) r = r * (a - b + i) / i;
    return r;
}

/* F = sum over degrees m = 0..n-1 of binom(d+m-1, m). */
long oracle_num_features(int d, int n) {
    if (d < 1 || n < 1) return -1;
    long F = 0;
    for (int m = 0; m < n; ++m) F += binom_l(d + m - 1, m);
    return F;
}

/* Degree-major table; inside a degree, non-decreasing tuples in lexicographic
 * order.  deg[F]; idx[F * width] with width = max(n-1, 1), unused slots -1;
 * w[F] = sqrt(m! / prod(multiplicity!)).  Any output pointer may be NULL. */
int oracle_feature_table(int d, int n, int32_t* deg, int32_t* idx, double* w) {
    long F = oracle_num_features(d, n);
    if (F < 0) return -1;
    int width = n > 1 ? n - 1 : 1;
    long f = 0;
    int t[64];
    if (n - 1 > 64) return -1;
    for (int m = 0; m < n; ++m) {
        for (int p = 0; p < m; ++p) t[p] = 0;
        for (;;) {
            if (deg) deg[f] = m;
            if (idx) {
                for (int p = 0; p < width; ++p) idx[f * width + p] = p < m ? t[p] : -1;
            }
            if (w) {
                double mf = 1.0, den = 1.0;
                for (int p = 1; p <= m; ++p) mf *= p;
                int run = 1;
                for (int p = 1; p <= m; ++p) {
                    if (p < m && t[p] == t[p - 1]) {
                        ++run;
                    } else {
                        for (int r = 2; r <= run; ++r) den *= r;
                        run = 1;
                    }
                }
                w[f] = sqrt(mf / den);
            }
            ++f;
            /* next non-decreasing tuple: bump the rightmost slot below d-1 and
             * copy its new value to every slot on its right */
            int p = m - 1;
            while (p >= 0 && t[p] == d - 1) --p;
            if (p < 0) break;
            t[p] += 1;
            for (int r = p + 1; r < m; ++r) t[r] = t[p];
        }
    }
    return f == F ? 0 : -2;
}

typedef struct {
    long F;
    int width;
    int32_t* deg;
    int32_t* idx;
    double* w;
} table_t;

static int table_make(table_t* tb, int d, int n) {
    tb->deg = NULL;
    tb->idx = NULL;
    tb->w = NULL;
    tb->F = oracle_num_features(d, n);
    if (tb->F < 0) return -1;
    tb->width = n > 1 ? n - 1 : 1;
    tb->deg = (int32_t*)malloc(sizeof(int32_t) * tb->F);
    tb->idx = (int32_t*)malloc(sizeof(int32_t) * tb->F * tb->width);
    tb->w = (double*)malloc(sizeof(double) * tb->F);
    if (!tb->deg || !tb->idx || !tb->w) return -3;
    return oracle_feature_table(d, n, tb->deg, tb->idx, tb->w);
}

static void table_free(table_t* tb) {
    free(tb->deg);
    free(tb->idx);
    free(tb->w);
}

/* phi(x) into out[F]; when query != 0 the factor tau^m/m! is applied. */
static void phi(const table_t* tb, const double* x, double tau, int query, double* out) {
    for (long f = 0; f < tb->F; ++f) {
        int m = tb->deg[f];
        double p = tb->w[f];
        for (int s = 0; s < m; ++s) p *= x[tb->idx[f * tb->width + s]];
        if (query) {
            double c = 1.0;
            for (int s = 1; s <= m; ++s) c *= tau / s;
            p *= c;
        }
        out[f] = p;
    }
}

/* Token-by-token recursion over BH independent heads.
 * q,k: [BH][N][d]; v: [BH][N][dv]; state_in (nullable) / state_out
 * (nullable): [BH][F][dv+1]; out: [BH][N][dv].  Update, then read out. */
int oracle_recurrent(long BH, long N, int d, int dv, int n, double tau,
                     const double* q, const double* k, const double* v,
                     const double* state_in, double* out, double* state_out, int nthreads) {
    table_t tb;
    if (BH < 0 || N < 0 || d < 1 || dv < 1 || n < 1) return -1;
    if (table_make(&tb, d, n) != 0) { table_free(&tb); return -1; }
    const long F = tb.F;
    const int Dv = dv + 1;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (long h = 0; h < BH; ++h) {
        double* S = (double*)malloc(sizeof(double) * F * Dv);
        double* pk = (double*)malloc(sizeof(double) * F);
        double* pq = (double*)malloc(sizeof(double) * F);
        double* y = (double*)malloc(sizeof(double) * Dv);
        if (!S || !pk || !pq || !y) { err |= 1; free(S); free(pk); free(pq); free(y); continue; }
        if (state_in) memcpy(S, state_in + h * F * Dv, sizeof(double) * F * Dv);
        else memset(S, 0, sizeof(double) * F * Dv);
        for (long i = 0; i < N; ++i) {
            const double* qi = q + (h * N + i) * d;
            const double* ki = k + (h * N + i) * d;
            const double* vi = v + (h * N + i) * dv;
            phi(&tb, ki, tau, 0, pk);
            phi(&tb, qi, tau, 1, pq);
            for (long f = 0; f < F; ++f) {
                double* row = S + f * Dv;
                for (int c = 0; c < dv; ++c) row[c] += pk[f] * vi[c];
                row[dv] += pk[f];
            }
            for (int c = 0; c < Dv; ++c) y[c] = 0.0;
            for (long f = 0; f < F; ++f) {
                const double* row = S + f * Dv;
                for (int c = 0; c < Dv; ++c) y[c] += pq[f] * row[c];
            }
            double* oi = out + (h * N + i) * dv;
            for (int c = 0; c < dv; ++c) oi[c] = y[c] / y[dv];
        }
        if (state_out) memcpy(state_out + h * F * Dv, S, sizeof(double) * F * Dv);
        free(S); free(pk); free(pq); free(y);
    }
    table_free(&tb);
    return err ? -3 : 0;
}

/* Pairwise (quadratic) form for selected rows: for each r, head hs[r] and
 * position rows[r], o = sum_{j<=i} K(tau q_i.k_j) v_j / sum_{j<=i} K(...).
 * q,k: [Hs][N][d]; v: [Hs][N][dv]; out: [R][dv]; den (nullable): [R]. */
int oracle_direct_rows(long N, int d, int dv, int n, double tau,
                       const double* q, const double* k, const double* v,
                       long R, const int64_t* hs, const int64_t* rows,
                       double* out, double* den, int nthreads) {
    if (N < 0 || d < 1 || dv < 1 || n < 1 || R < 0) return -1;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 4) reduction(| : err)
    for (long r = 0; r < R; ++r) {
        long h = hs[r], i = rows[r];
        if (i < 0 || i >= N || h < 0) { err |= 1; continue; }
        const double* qi = q + (h * N + i) * d;
        double* num = out + r * dv;
        for (int c = 0; c < dv; ++c) num[c] = 0.0;
        double dd = 0.0;
        for (long j = 0; j <= i; ++j) {
            const double* kj = k + (h * N + j) * d;
            const double* vj = v + (h * N + j) * dv;
            double x = 0.0;
            for (int s = 0; s < d; ++s) x += qi[s] * kj[s];
            x *= tau;
            /* sum_{m<n} x^m/m! by Horner: 1 + x(1 + x/2(1 + x/3(...))) */
            double wgt = 1.0;
            for (int m = n - 1; m >= 1; --m) wgt = 1.0 + wgt * x / m;
            for (int c = 0; c < dv; ++c) num[c] += wgt * vj[c];
            dd += wgt;
        }
        for (int c = 0; c < dv; ++c) num[c] /= dd;
        if (den) den[r] = dd;
    }
    return err ? -1 : 0;
}

/* Sum over a token range of phi(k_j)[v_j|1]^T, for selected heads: the state
 * after tokens [0, N) from zero, accumulated in float64.  Same layout as
 * state_out above. */
int oracle_state(long BH, long N, int d, int dv, int n,
                 const double* k, const double* v, double* state_out, int nthreads) {
    table_t tb;
    if (BH < 0 || N < 0 || d < 1 || dv < 1 || n < 1) return -1;
    if (table_make(&tb, d, n) != 0) { table_free(&tb); return -1; }
    const long F = tb.F;
    const int Dv = dv + 1;
    int err = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (long h = 0; h < BH; ++h) {
        double* pk = (double*)malloc(sizeof(double) * F);
        if (!pk) { err |= 1; continue; }
        double* S = state_out + h * F * Dv;
        memset(S, 0, sizeof(double) * F * Dv);
        for (long j = 0; j < N; ++j) {
            const double* kj = k + (h * N + j) * d;
            const double* vj = v + (h * N + j) * dv;
            phi(&tb, kj, 0.0, 0, pk);
            for (long f = 0; f < F; ++f) {
                double* row = S + f * Dv;
                for (int c = 0; c < dv; ++c) row[c] += pk[f] * vj[c];
                row[dv] += pk[f];
            }
        }
        free(pk);
    }
    table_free(&tb);
    return err ? -3 : 0;
}
