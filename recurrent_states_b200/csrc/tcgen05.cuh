// Inline-PTX wrappers for the sm_100a tensor cores (tcgen05) and the
// shared-memory matrix descriptors they read.  Only the forms this library
// uses: one CTA (cta_group::1), kind::f16 with bf16 operands read from shared
// memory and an fp32 accumulator in tensor memory (TMEM).
//
// Operand layouts (no swizzle, "interleaved" canonical layouts).  A core
// matrix is 8 rows of 16 bytes (8 bf16) stored contiguously (128 bytes).
//  * K-major operand X[R][K] (K contiguous within a core row): element (r, k)
//    at (r/8)*SBO + (k/8)*LBO + (r%8)*16 + (k%8)*2 bytes.
//  * MN-major operand Y[K][MN] (MN contiguous within a core row): element
//    (k, x) at (x/8)*SBO + (k/8)*LBO + (k%8)*16 + (x%8)*2 bytes.
// In both, SBO is the stride between 8-element groups of the M/N dimension
// and LBO the stride between 8-element groups of K.  One MMA consumes K = 16
// (two K groups); the next K step starts 2*LBO bytes further on.
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace ta {
namespace tc {

// ---------------------------------------------------------------- descriptors

// Shared-memory matrix descriptor: start address, LBO, SBO (all >> 4),
// the sm_100 descriptor version (1) and layout type 0 (no swizzle).
__device__ __forceinline__ uint64_t smem_desc(const void* start, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    const uint32_t a = ptx::smem_u32(start);
    uint64_t d = 0;
    d |= (uint64_t)((a >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;  // version
    return d;
}

// Swizzled layouts (the forms TMA writes with CU_TENSOR_MAP_SWIZZLE_*):
// rows of 32, 64 or 128 bytes whose 16-byte chunks are XOR-permuted by
// address bits 7.. (chunk c of row r lands at chunk c ^ sw(r)); the atom
// base must be 1024-byte aligned.  K-major: LBO is unused, SBO = 8 rows.
// MN-major (128 B): LBO = stride between 64-element atoms along MN, SBO =
// stride between groups of 8 K rows.
enum : uint32_t { kSwizzleNone = 0, kSwizzle128 = 2, kSwizzle64 = 4, kSwizzle32 = 6 };

__device__ __forceinline__ uint64_t smem_desc_sw(const void* start, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                                 uint32_t layout) {
    return smem_desc(start, lbo_bytes, sbo_bytes) | ((uint64_t)layout << 61);
}

// Chunk permutation of row r in a swizzled layout with row_bytes-wide rows.
__host__ __device__ constexpr uint32_t swizzle_of_row(uint32_t r, uint32_t row_bytes) {
    return ((r * row_bytes) >> 7) & (row_bytes / 16 - 1);
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 accumulator,
// M x N tile, each operand K-major (0) or MN-major (1).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
    return (1u << 4)                      // D format: f32
           | (1u << 7)                    // A format: bf16
           | (1u << 10)                   // B format: bf16
           | ((uint32_t)a_mn_major << 15) //
           | ((uint32_t)b_mn_major << 16) //
           | ((uint32_t)(N >> 3) << 17)   //
           | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of row r, 8-element K group `kgroup` in a K-major operand with
// LBO = 128 (K groups of a row group contiguous) and row-group stride sbo.
__device__ __forceinline__ uint32_t kmaj(int r, int kgroup, uint32_t sbo) {
    return (uint32_t)(r >> 3) * sbo + (uint32_t)kgroup * 128u + (uint32_t)(r & 7) * 16u;
}

// Byte offset of K row k, 8-element MN group `ngroup` in an MN-major operand
// with SBO = 128 (MN groups of a K group contiguous) and K-group stride lbo.
__device__ __forceinline__ uint32_t mnmaj(int k, int ngroup, uint32_t lbo) {
    return (uint32_t)ngroup * 128u + (uint32_t)(k >> 3) * lbo + (uint32_t)(k & 7) * 16u;
}

// ---------------------------------------------------------------- TMEM

// Allocates ncols TMEM columns (power of two >= 32); the whole warp calls it.
// The base address is written to *slot (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(ptx::smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---------------------------------------------------------------- MMA

// D[tmem] (+)= A[smem] x B[smem]; accumulate when acc != 0.  One thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t acc) {
    const uint32_t mask0 = 0, mask1 = 0, mask2 = 0, mask3 = 0;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
        "}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc), "r"(mask0), "r"(mask1), "r"(mask2), "r"(mask3)
        : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem] (A K-major in TMEM: lane = row, each 32-bit
// column two consecutive bf16 of K, low half first).  One thread.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t acc) {
    const uint32_t mask0 = 0, mask1 = 0, mask2 = 0, mask3 = 0;
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t"
        "}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(acc), "r"(mask0), "r"(mask1), "r"(mask2), "r"(mask3)
        : "memory");
}

// Arrives once on the mbarrier when every MMA this thread issued so far has
// completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     ptx::smem_u32(bar))
                 : "memory");
}

// ---------------------------------------------------------------- TMEM -> registers

// 32 consecutive columns of this thread's lane (warp w reads lanes 32*(w%4)..).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&r)[32]) {
    uint32_t u[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]),
          "=r"(u[23]), "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]),
          "=r"(u[30]), "=r"(u[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __uint_as_float(u[i]);
}

// 16 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&r)[16]) {
    uint32_t u[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
}

// One column of this thread's lane.
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t u;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(u) : "r"(taddr) : "memory");
    return __uint_as_float(u);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- registers -> TMEM

// 32 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&u)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15]), "r"(u[16]), "r"(u[17]),
        "r"(u[18]), "r"(u[19]), "r"(u[20]), "r"(u[21]), "r"(u[22]), "r"(u[23]), "r"(u[24]), "r"(u[25]), "r"(u[26]),
        "r"(u[27]), "r"(u[28]), "r"(u[29]), "r"(u[30]), "r"(u[31])
        : "memory");
}

// 16 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&u)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}

// 8 consecutive columns of this thread's lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&u)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- bf16 hi/lo split

// x ~= hi + lo with hi = x truncated to bf16 (its top 16 bits) and
// lo = bf16(x - hi), the remainder being exact in fp32: 16 significant bits
// (representation error below 2^-17 |x|).  The hi pair is a byte permute and
// the lo pair one conversion, so a pair costs one conversion instruction.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const uint32_t b0 = __float_as_uint(x0), b1 = __float_as_uint(x1);
    const float r0 = x0 - __uint_as_float(b0 & 0xffff0000u);
    const float r1 = x1 - __uint_as_float(b1 & 0xffff0000u);
    hi = __byte_perm(b0, b1, 0x7632);
    const __nv_bfloat162 l = __floats2bfloat162_rn(r0, r1);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Packs 8 floats as hi and lo bf16 vectors (16 bytes each).
__device__ __forceinline__ void split8(const float* x, uint4& hi, uint4& lo) {
    split2(x[0], x[1], hi.x, lo.x);
    split2(x[2], x[3], hi.y, lo.y);
    split2(x[4], x[5], hi.z, lo.z);
    split2(x[6], x[7], hi.w, lo.w);
}

}  // namespace tc
}  // namespace ta
