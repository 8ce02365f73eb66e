// 5th-generation tensor core (tcgen05) helpers for sm_100a: tensor-memory
// allocation, block-scaled MMA (kind::mxf8f6f4), bf16 MMA (kind::f16),
// scale-factor copies into
// tensor memory, tensor-memory loads, and the shared-memory matrix
// descriptors these instructions read.
#pragma once

#include "ptx.cuh"

namespace moe {

// ---- tensor memory (TMEM): 128 lanes x 512 columns of 32 bits per SM ----
// Address format: lane in bits 31..16, column in bits 15..0.

// Warp-wide: allocates `ncols` columns (a power of two >= 32) and writes the
// base address to shared memory.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Order tcgen05 operations against thread synchronisation (mbarriers, bar.sync).
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrives once on `bar` when every tcgen05.mma / tcgen05.cp this thread issued
// before it has completed.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 rows x 16 bytes of scale factors from shared memory, broadcast to the
// same rows of all four 32-lane quarters of TMEM (4 columns from `taddr`).
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// D[M][N] (+)= (A[M][K] * sfa) . (B[N][K] * sfb)^T with K = 32, fp32 accumulate
// in TMEM; A and B in shared memory (descriptors), E8M0 scale factors in TMEM.
__device__ __forceinline__ void tc_mma_mx(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// The same for kind::mxf4: A and B packed E2M1 (two per byte), K = 64, two
// E8M0 scale factors per row (scale_vec::2X: bytes sf id and sf id + 1 of the
// TMEM scale word, sf id 0 or 2).
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// D[M][N] (+)= A[M][K] . B[N][K]^T with K = 16 bf16 elements, fp32 accumulate
// in TMEM; A and B in shared memory (descriptors).
__device__ __forceinline__ void tc_mma_bf16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same with A in tensor memory (lane m = row m of A, K-major, two bf16 per
// 32-bit column: K = 16 is 8 columns from a_tmem); B from shared memory.
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Thread i of the warp writes TMEM lane (lane field of taddr) + i, columns
// taddr .. taddr + 31, from r[0 .. 31].
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Thread i of the warp reads TMEM lane (lane field of taddr) + i, columns
// taddr .. taddr + 31 (one 32-bit value per column).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---- shared-memory matrix descriptors ----
// Fields: start address >> 4 (bits 0..13), leading byte offset >> 4
// (16..29), stride byte offset >> 4 (32..45), version 1 (46..47), layout
// type (61..63: 0 none, 2 = 128-byte swizzle).

// K-major operand tile written by a 128-byte-swizzled TMA box: rows of 128
// bytes, 8-row groups 1024 bytes apart. The tile must start 1024-aligned;
// advancing K by 32 one-byte elements adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t sdesc_sw128(const void *p) {
    const uint64_t a = smem_u32(p);
    return ((a >> 4) & 0x3FFFull) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}

// Scale-factor atom for tcgen05.cp 32x128b: 32 rows of 16 bytes, contiguous
// (8-row core matrices 128 bytes apart), no swizzle.
__device__ __forceinline__ uint64_t sdesc_sf(const void *p) {
    const uint64_t a = smem_u32(p);
    return ((a >> 4) & 0x3FFFull) | (8ull << 32) | (1ull << 46);
}

// Instruction descriptor of the block-scaled kinds with E8M0 scales (bit 23),
// both operands K-major, dense K (32 for kind::mxf8f6f4, 64 for kind::mxf4:
// bit 31 clear). Formats: mxf8f6f4 0 = E4M3, 5 = E2M1; mxf4 1 = E2M1. The
// scale-factor byte ids (which of the 4 bytes of each TMEM word) are or-ed in
// per K step.
__host__ __device__ constexpr uint32_t idesc_mx(int a_fmt, int b_fmt, int M, int N) {
    return (uint32_t)(a_fmt & 7) << 7 | (uint32_t)(b_fmt & 7) << 10 | (uint32_t)(N >> 3) << 17 | 1u << 23 |
           (uint32_t)(M >> 4) << 24;
}
// Instruction descriptor of kind::f16 with bf16 A and B (both K-major) and an
// fp32 accumulator: D format 1 (bits 4..5), A and B format 1 = bf16 (bits
// 7..9, 10..12), N / 8 (bits 17..22), M / 16 (bits 24..28).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return 1u << 4 | 1u << 7 | 1u << 10 | (uint32_t)(N >> 3) << 17 | (uint32_t)(M >> 4) << 24;
}
__device__ __forceinline__ uint32_t idesc_sf_ids(uint32_t idesc, uint32_t a_id, uint32_t b_id) {
    return idesc | (b_id & 3u) << 4 | (a_id & 3u) << 29;
}

}  // namespace moe
