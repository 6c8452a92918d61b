// Phase markers for timing the inside of a kernel.  They compile to nothing
// unless TA_PHASE_PROBE is defined, in which case the including translation
// unit must define TA_PHASE_KERNELS and provide
// `__device__ unsigned long long g_ta_phase[TA_PHASE_KERNELS * 65536 * 16]`;
// each marker then records %globaltimer for the block (slot i of 16, kernel
// k), skipping any index outside that array.
#pragma once

#ifdef TA_PHASE_PROBE
#define TA_PHASE(k, i, cond)                                                                          \
    do {                                                                                              \
        const unsigned b_ = blockIdx.y * gridDim.x + blockIdx.x;                                      \
        if ((cond) && (k) < TA_PHASE_KERNELS && b_ < 65536u && (i) < 16) {                            \
            unsigned long long t_;                                                                    \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                                    \
            g_ta_phase[((size_t)(k) * 65536 + b_) * 16 + (i)] = t_;                                   \
        }                                                                                             \
    } while (0)
// Cycle accumulators for the inside of a loop: TA_PHASE_VARS declares
// counters, TA_PHASE_T0 takes a start time, TA_PHASE_ACC adds the cycles
// since it to a counter, TA_PHASE_PUT stores a counter into slot i.
#define TA_PHASE_VARS(...) unsigned long long __VA_ARGS__
#define TA_PHASE_T0(t) (t) = clock64()
#define TA_PHASE_ACC(acc, t) (acc) += clock64() - (t)
#define TA_PHASE_PUT(k, i, cond, val)                                                                 \
    do {                                                                                              \
        const unsigned b_ = blockIdx.y * gridDim.x + blockIdx.x;                                      \
        if ((cond) && (k) < TA_PHASE_KERNELS && b_ < 65536u && (i) < 16)                             \
            g_ta_phase[((size_t)(k) * 65536 + b_) * 16 + (i)] = (val);                                \
    } while (0)
#else
#define TA_PHASE(k, i, cond) \
    do {                     \
    } while (0)
#define TA_PHASE_VARS(...)
#define TA_PHASE_T0(t)
#define TA_PHASE_ACC(acc, t)
#define TA_PHASE_PUT(k, i, cond, val) \
    do {                              \
    } while (0)
#endif
