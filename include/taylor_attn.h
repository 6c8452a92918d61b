/*
 * taylor_attn.h -- C ABI of libtaylor_attn.so: causal attention whose
 * exponential kernel is replaced by its truncated Taylor series, evaluated
 * through n additive recurrent states, on NVIDIA B200 (sm_100a).
 *
 * Method: "Expanding Attention: A Taylor-Series Route to Linear-Time
 * Transformers with a Fixed Number of Recurrent States" (arXiv 2610.20637),
 * abstract.  With x = tau * q.k for unit-norm q, k (the caller normalises),
 *     K(q, k) = sum_{m=0}^{n-1} x^m / m!
 *             = sum_m (tau^m / m!) <phi_m(q), phi_m(k)>,
 * where phi_m packs the binom(d_k+m-1, m) monomials x_{i1}...x_{im},
 * i1 <= ... <= im, each times sqrt(m!/alpha!) (alpha = index multiplicities).
 * The causal history is the state S = sum_j phi(k_j) [v_j | 1]^T (F rows,
 * d_v + 1 columns, F = binom(d_k+n-1, n-1)), and
 *     o_i = y[0:d_v] / y[d_v],   y = (c (.) phi(q_i))^T S_{<=i},
 * c = tau^m/m! per feature.  Causality is inclusive (token i sees j <= i).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Sizes: 1 <= n <= 5, 1 <= d_k <= 64, 4 <= d_v <= 256 with d_v % 4 == 0,
 *   B, H, N >= 0 with B*H*N < 2^31 tokens.  Anything else returns
 *   TAYLOR_ERR_UNSUPPORTED (sizes out of range) or TAYLOR_ERR_INVALID_ARG
 *   (negative sizes, NULL required pointers, non-finite tau).
 * - Tensors are dense, row-major, caller-owned DEVICE pointers on the current
 *   device, aligned to 16 bytes (else TAYLOR_ERR_MISALIGNED):
 *     q, k  [B][H][N][d_k]   bf16 (the plain calls) or fp32 (the _f32 calls)
 *     v     [B][H][N][d_v]   same dtype as q, k
 *     out   [B][H][N][d_v]   fp32
 *     state [B][H][stride]   fp32, stride = taylor_attn_state_stride(); per
 *           head: S_v[F][d_v] row-major, then z[F] (the ones column of
 *           [v | 1]), then zero padding up to stride (a multiple of 32
 *           floats).  The state holds pure phi(k): it does not depend on tau.
 *   Feature f follows taylor_attn_feature_index(): degree-major, and inside a
 *   degree the non-decreasing index tuples in lexicographic order.
 * - Every call is asynchronous on `stream` (may be 0, the legacy default
 *   stream) and returns after enqueueing.  Status TAYLOR_OK means the work
 *   was enqueued; launch failures are reported as TAYLOR_ERR_CUDA.  Calls
 *   keep no state between them and are safe from several host threads.
 * - No epsilon in the quotient: IEEE fp32 division on the CUDA-core paths
 *   and in decode, a multiplication by the correctly rounded reciprocal
 *   (within 1.5 ulp of the quotient) in the tensor-core prefill.  For even n
 *   the denominator can reach zero for un-normalised inputs and the output is
 *   then inf/nan.
 *
 * The n = 3 state also serves a second read-out, the mean-centred Taylor
 * expansion of softmax (taylor_attn_centred_decode, below).
 */
#ifndef TAYLOR_ATTN_H
#define TAYLOR_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define TAYLOR_API __attribute__((visibility("default")))
#else
#define TAYLOR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum taylor_attn_status {
    TAYLOR_OK = 0,
    TAYLOR_ERR_INVALID_ARG = -1,   /* NULL pointer, negative size, bad tau   */
    TAYLOR_ERR_UNSUPPORTED = -2,   /* n, d_k, d_v or total size out of range  */
    TAYLOR_ERR_MISALIGNED = -3,    /* a pointer not 16-byte aligned           */
    TAYLOR_ERR_CUDA = -4,          /* a CUDA runtime call or launch failed    */
    TAYLOR_ERR_OUT_OF_MEMORY = -5, /* stream-ordered workspace alloc failed   */
    TAYLOR_ERR_SCRATCH_LIMIT = -6, /* work exceeds the fixed no-alloc scratch */
    TAYLOR_ERR_TIMEOUT = -7        /* a bounded device-side wait ran out      */
};

/* Short English text for a status code (static storage, never NULL). */
TAYLOR_API const char* taylor_attn_strerror(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
TAYLOR_API int taylor_attn_version(void);

/* F = sum_{m<n} binom(d_k+m-1, m) = binom(d_k+n-1, n-1), the packed width
 * of phi (abstract: the m-th state is binom(d+m-1, m) wide).  Returns -1
 * when (d_k, n) is outside the supported range.  Host only. */
TAYLOR_API int64_t taylor_attn_num_features(int d_k, int n);

/* Floats per head of a state: F*(d_v+1) rounded up to a multiple of 32.
 * At d_k = 16, d_v = 64, n = 3: F*(d_v+1) = 9,945 (the abstract's count of
 * elements per head), stride 9,952.  Returns -1 when unsupported.  Host only. */
TAYLOR_API int64_t taylor_attn_state_stride(int d_k, int d_v, int n);

/* The packed feature order, written to HOST memory: deg[F] receives the
 * degree m of each feature, idx[F * max(n-1, 1)] its indices i1 <= ... <= im
 * followed by -1 padding.  Returns TAYLOR_OK or an error code. */
TAYLOR_API int taylor_attn_feature_index(int d_k, int n, int32_t* deg, int32_t* idx);

/* Step 1 of the path, exposed on its own (abstract: tensor-power
 * factorisation).  For T vectors x[T][d_k] (fp32, device) writes
 * phi[T][F] (fp32, device), phi_f(x) = sqrt(m!/alpha!) prod_t x[i_t]; with
 * query_side != 0 each feature is also multiplied by tau^m/m!. */
TAYLOR_API int taylor_attn_feature_map(const float* x, float* phi, int64_t T, int d_k, int n,
                            float tau, int query_side, cudaStream_t stream);

/* Causal prefill from the empty state (abstract: prefill admits a parallel
 * scan because states are additive across chunks).  q, k, v are bf16.
 * Writes out[B][H][N][d_v] and, when state_out != NULL, the state after all
 * N tokens.  N == 0 writes a zero state.  Takes stream-ordered workspace on
 * `stream` (one fp32 state per 64-128 tokens per head) from a memory pool the
 * library creates per device; freed workspace stays cached in that pool for
 * later calls, up to the larger of 1 GiB and the largest workspace one call
 * has needed (taylor_attn_release_workspace returns it).
 * TAYLOR_ERR_OUT_OF_MEMORY if the workspace cannot be had; accumulation is
 * fp32. */
TAYLOR_API int taylor_attn_prefill(const void* q, const void* k, const void* v, float* out,
                        float* state_out, int B, int H, int N, int d_k, int d_v, int n,
                        float tau, cudaStream_t stream);

/* Same as taylor_attn_prefill with fp32 q, k, v; every product and sum is
 * fp32 on CUDA cores (no reduced-precision tensor-core operand). */
TAYLOR_API int taylor_attn_prefill_f32(const float* q, const float* k, const float* v, float* out,
                            float* state_out, int B, int H, int N, int d_k, int d_v, int n,
                            float tau, cudaStream_t stream);

/* Causal prefill that continues a sequence from a carried state: tokens
 * 0..N-1 here are positions P..P+N-1 of a sequence whose first P tokens
 * produced state_in [B][H][stride] (by a prefill, decodes or merges).  Each
 * output attends to the carried prefix through state_in and to the new
 * tokens as taylor_attn_prefill does; state_out (may be NULL, may alias
 * state_in) receives state_in plus the new tokens' state (abstract: states
 * are additive across chunks, so prefill can resume from a chunk boundary).
 * q, k, v bf16; workspace and errors as taylor_attn_prefill.  With N <= 16,
 * d_v in {16, 32, 64, 128} and at most 1,024 features this is batched
 * multi-token decode: one kernel reads and writes each head's state once
 * and allocates no workspace. */
TAYLOR_API int taylor_attn_prefill_from_state(const void* q, const void* k, const void* v,
                                              const float* state_in, float* out, float* state_out,
                                              int B, int H, int N, int d_k, int d_v, int n, float tau,
                                              cudaStream_t stream);

/* taylor_attn_prefill_from_state with fp32 q, k, v (CUDA-core fp32 path). */
TAYLOR_API int taylor_attn_prefill_from_state_f32(const float* q, const float* k, const float* v,
                                                  const float* state_in, float* out, float* state_out,
                                                  int B, int H, int N, int d_k, int d_v, int n,
                                                  float tau, cudaStream_t stream);

/* Returns the prefill workspace cached in the current device's pool to the
 * driver (synchronises the device first). */
TAYLOR_API int taylor_attn_release_workspace(void);

/* One new token per (b, h) against carried states (abstract: per-token
 * decoding latency is constant in N).  q, k [B][H][d_k] and v [B][H][d_v]
 * are bf16; state_inout [B][H][stride] is read and overwritten in place with
 * S + phi(k)[v | 1]^T; out [B][H][d_v] receives the read-out after that
 * update.  No workspace. */
TAYLOR_API int taylor_attn_decode(const void* q, const void* k, const void* v, float* state_inout,
                       float* out, int B, int H, int d_k, int d_v, int n, float tau,
                       cudaStream_t stream);

/* taylor_attn_decode with fp32 q, k, v. */
TAYLOR_API int taylor_attn_decode_f32(const float* q, const float* k, const float* v, float* state_inout,
                           float* out, int B, int H, int d_k, int d_v, int n, float tau,
                           cudaStream_t stream);

/* One new token per (b, h) for causal attention with the mean-centred
 * Taylor expansion of softmax instead of the truncated exponential kernel
 * (Su Jianlin, "Taylor expansions of logsumexp and softmax", kexue.fm
 * translation 11814, sections "Calculating the Gradient" and "Linear
 * Attention"): the row of token i weights v_j, j <= i, by
 * (1 + y_j + (y_j^2 - mean(y^2))/2) / (i + 1) with y_j = tau q.(k_j - kbar)
 * and kbar the mean of those keys; order 1 drops the square term.  Weights
 * are used as they are (they sum to one; no clamp of negative ones).
 * The carried state is the n = 3 Taylor state of the same keys and values
 * ([B][H][taylor_attn_state_stride(d_k, d_v, 3)], layout as
 * taylor_attn_decode; its degree-0..2 blocks hold every prefix sum the
 * expansion needs), updated in place with S + phi(k)[v | 1]^T exactly as
 * taylor_attn_decode with n = 3 would; it can come from taylor_attn_prefill
 * with n = 3 and stays valid for both read-outs.  q, k [B][H][d_k], v
 * [B][H][d_v] bf16 (the _f32 variant: fp32); out [B][H][d_v] fp32.  order is
 * 1 or 2 (else TAYLOR_ERR_UNSUPPORTED); d_k in 1..64, d_v a multiple of 4 up
 * to 256; pointers 16-byte aligned.  No workspace. */
TAYLOR_API int taylor_attn_centred_decode(const void* q, const void* k, const void* v, float* state_inout,
                                          float* out, int B, int H, int d_k, int d_v, int order, float tau,
                                          cudaStream_t stream);

/* taylor_attn_centred_decode with fp32 q, k, v. */
TAYLOR_API int taylor_attn_centred_decode_f32(const float* q, const float* k, const float* v,
                                              float* state_inout, float* out, int B, int H, int d_k, int d_v,
                                              int order, float tau, cudaStream_t stream);

/* Causal prefill with the mean-centred Taylor expansion of softmax (the same
 * method and readings as taylor_attn_centred_decode: Su Jianlin, "Taylor
 * expansions of logsumexp and softmax", kexue.fm translation 11814, sections
 * "Calculating the Gradient" and "Linear Attention").  Row i weights v_j,
 * j <= i, by (1 + y_j + (y_j^2 - mean(y^2))/2) / (i + 1), y_j = tau
 * q_i.(k_j - kbar_i), kbar_i the mean of k_0..k_i; order 1 drops the square
 * term.  q, k [B][H][N][d_k], v [B][H][N][d_v] bf16 (the _f32 variant:
 * fp32); out [B][H][N][d_v] fp32.  state_out (may be NULL) receives the n = 3
 * Taylor state of the N tokens ([B][H][taylor_attn_state_stride(d_k, d_v,
 * 3)]), from which taylor_attn_centred_decode (or taylor_attn_decode with
 * n = 3) continues.  The three per-degree read-outs sum_j (q_i.k_j)^m [v_j | 1]
 * (m = 0, 1, 2) are accumulated apart, pairwise inside a chunk or token group
 * and through the exclusive n = 3 state before it, and combined per column in
 * fp32: with bf16 inputs, d_k 16 and d_v 64 on the tensor cores (hi/lo bf16
 * operands, fp32 accumulators), else in fp32 on CUDA cores.  order is 1 or 2
 * (else TAYLOR_ERR_UNSUPPORTED); sizes, alignment and workspace as
 * taylor_attn_prefill. */
TAYLOR_API int taylor_attn_centred_prefill(const void* q, const void* k, const void* v, float* out,
                                           float* state_out, int B, int H, int N, int d_k, int d_v, int order,
                                           float tau, cudaStream_t stream);

/* taylor_attn_centred_prefill with fp32 q, k, v. */
TAYLOR_API int taylor_attn_centred_prefill_f32(const float* q, const float* k, const float* v, float* out,
                                               float* state_out, int B, int H, int N, int d_k, int d_v,
                                               int order, float tau, cudaStream_t stream);

/* out = a + b over B*H states (abstract: states are additive across chunks,
 * so the state of a concatenation is the sum of the parts' states).  out may
 * alias a or b.  No workspace. */
TAYLOR_API int taylor_attn_state_merge(const float* a, const float* b, float* out, int B, int H,
                            int d_k, int d_v, int n, cudaStream_t stream);

/* taylor_attn_prefill_f32 for callers that cannot allocate device memory
 * (a plugin whose host framework owns all device memory, a serving loop that
 * reserves memory up front and must not see an allocation fail mid-step).
 * The paper has no counterpart: this is a deployment variant.  The scratch
 * for the scan across token groups lives in one fixed file-scope device array
 * of taylor_attn_prefill_noalloc_scratch_floats() floats (16 MiB), held on
 * every GPU that loads the library until the process exits; the call makes no
 * cudaMalloc/cudaFree or other allocating call.  Work needing more scratch
 * than that (B*H * groups * stride floats; the B1 H8 N4096 d_k16 d_v64 n3
 * shape needs about 2.5 million) returns TAYLOR_ERR_SCRATCH_LIMIT before any launch.
 * The first call on a device looks up the array's device address; CUDA loads
 * device code lazily, so that first call is also the one that brings the
 * array's 16 MiB onto the device, and it can fail with
 * TAYLOR_ERR_OUT_OF_MEMORY when the device is already full.  Make it during
 * set-up, before reserving the rest of the device's memory and before any
 * stream capture; a failed first call is retried by the next one.  All calls
 * on a device share the array: calls that overlap on the GPU race and must be
 * serialised by the caller.  Same arguments, layouts and results as
 * taylor_attn_prefill_f32. */
TAYLOR_API int taylor_attn_prefill_f32_noalloc(const float* q, const float* k, const float* v,
                                               float* out, float* state_out, int B, int H, int N,
                                               int d_k, int d_v, int n, float tau,
                                               cudaStream_t stream);

/* Size in floats of the fixed scratch used by taylor_attn_prefill_f32_noalloc. */
TAYLOR_API int64_t taylor_attn_prefill_noalloc_scratch_floats(void);

/* Kernels that wait on asynchronous copies (mbarriers) bound every wait;
 * when a bound runs out the kernel sets a bit in a device error word and
 * returns early (its outputs are then incomplete).  This call reads that word
 * for the current device (a synchronous device-to-host copy that waits for
 * all prior work), stores it in *flags, clears it when clear != 0, and
 * returns TAYLOR_ERR_TIMEOUT if any bit was set, else TAYLOR_OK.
 * Bits: 1 = decode state load, 2 = decode state store, 4 = prefill pipeline,
 * 8 = taylor_attn_selftest_bounded_wait. */
TAYLOR_API int taylor_attn_device_errors(int clear, unsigned int* flags);

/* Exercises the timeout path on the device: one block waits on an mbarrier
 * that nothing arrives on, gives up after `polls` polls (1 .. 2^20), sets bit
 * 8 of the error word and returns; the context stays usable. */
TAYLOR_API int taylor_attn_selftest_bounded_wait(unsigned int polls, cudaStream_t stream);

/* Opt-in kernel timing, for benchmarks.  With on != 0, every kernel this
 * library launches from the calling host thread is bracketed by two CUDA
 * events on its stream (not usable inside CUDA graph capture). */
TAYLOR_API int taylor_attn_timing_enable(int on);

/* Waits for the recorded events of the calling thread, clears them, and
 * writes up to max_kernels entries: names[64 * i] (NUL-terminated kernel
 * name), launches[i], total_ms[i] (summed device time).  Returns the number
 * of distinct kernels seen (may exceed max_kernels) or an error code. */
TAYLOR_API int taylor_attn_timing_read(int max_kernels, char* names, int* launches,
                                       float* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* TAYLOR_ATTN_H */
