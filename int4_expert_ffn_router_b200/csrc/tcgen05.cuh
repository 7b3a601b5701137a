// tcgen05.cuh -- thin wrappers over the sm_100a fifth-generation tensor-core
// instructions (PTX ISA 8.7: tcgen05.alloc/dealloc, tcgen05.mma, tcgen05.ld/st,
// tcgen05.commit, tcgen05 fences) and the descriptors they take.
//
// Encodings (PTX ISA, "Instruction descriptor" and "Shared memory descriptor"
// tables of the tcgen05 section):
//   instruction descriptor, kind::f16, dense:
//     bits 4-5 D format (1 = f32), bits 7-9 A format, bits 10-12 B format
//     (0 = f16, 1 = bf16), bit 15/16 A/B major (0 = K-major), bits 17-22 N/8,
//     bits 24-28 M/16.
//   shared memory matrix descriptor:
//     bits 0-13 start address / 16, bits 16-29 leading byte offset / 16,
//     bits 32-45 stride byte offset / 16, bits 46-47 version (1),
//     bits 49-51 base offset, bit 52 LBO mode, bits 61-63 swizzle
//     (2 = 128-byte swizzle).
// A K-major operand with 128-byte swizzling is stored as rows of 128 bytes
// (64 16-bit elements), eight rows forming a 1024-byte atom in which the
// 16-byte chunk c of row r sits at chunk position c ^ (r & 7); atoms follow
// each other at the stride byte offset (1024). One MMA consumes 16 elements
// (32 bytes) of K, so the k-th step advances the start address by 32 bytes.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace coli {

__device__ __forceinline__ uint32_t tc_idesc_f16(int n, bool bf16) {
    const uint32_t ab = bf16 ? 1u : 0u;
    return (1u << 4) | (ab << 7) | (ab << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// K-major, 128-byte swizzled operand at shared address `saddr` (1024-aligned
// atom base), atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t tc_sdesc_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Allocation (one full warp; the column count is a power of two >= 32).
__device__ __forceinline__ void tc_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Warp-converged forms: the whole warp executes them, one elected lane
// performs the operation (several times cheaper to issue than from a
// one-lane branch). tc_commit_elect arrives once on `bar` when every
// tcgen05.mma the electing thread issued so far has completed.
__device__ __forceinline__ void tc_commit_elect(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}
__device__ __forceinline__ void mbar_arrive_elect(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\t.reg .b64 st;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
        : "memory");
}

// The eight MMAs of two 64-input blocks into one accumulator, then one
// commit to each of three barriers: D[d] (+)= A[a + 8 j] * B[desc_j]^T for
// j = 0..7, where desc_j is b0 + 2 j (j < 4) or b1 + 2 (j - 4) (the start
// address advances 32 bytes per 16 inputs), the first MMA accumulating only
// if `accumulate` != 0; bar0..bar2 (shared addresses) each receive one
// arrival when the MMAs have completed. Warp-converged: a single elect, one
// lane issues everything.
__device__ __forceinline__ void tc_mma8_commit3(uint32_t d, uint32_t a, uint64_t b0, uint64_t b1, uint32_t idesc,
                                                uint32_t accumulate, uint32_t bar0, uint32_t bar1, uint32_t bar2) {
    asm volatile(
        "{\n\t.reg .pred e, p, t;\n\t.reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"
        ".reg .b64 d1, d2, d3, d5, d6, d7;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %5, 0;\n\tsetp.eq.b32 t, %5, %5;\n\t"
        "add.u32 a1, %1, 8;\n\tadd.u32 a2, %1, 16;\n\tadd.u32 a3, %1, 24;\n\tadd.u32 a4, %1, 32;\n\t"
        "add.u32 a5, %1, 40;\n\tadd.u32 a6, %1, 48;\n\tadd.u32 a7, %1, 56;\n\t"
        "add.s64 d1, %2, 2;\n\tadd.s64 d2, %2, 4;\n\tadd.s64 d3, %2, 6;\n\t"
        "add.s64 d5, %3, 2;\n\tadd.s64 d6, %3, 4;\n\tadd.s64 d7, %3, 6;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a1], d1, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a2], d2, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a3], d3, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a4], %3, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a5], d5, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a6], d6, %4, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [a7], d7, %4, t;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%7];\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%8];\n\t}" ::"r"(d),
        "r"(a), "l"(b0), "l"(b1), "r"(idesc), "r"(accumulate), "r"(bar0), "r"(bar1), "r"(bar2)
        : "memory");
}

// Thread i of the warp writes lane (taddr.lane + i), columns taddr.col .. +15.
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Thread i reads lane (taddr.lane + i), columns taddr.col .. +15; waits for
// the load inside the same statement so the registers are valid on return.
__device__ __forceinline__ void tc_ld16_wait(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

// TMA tile load: box at (x, y) of a 2D tensor map into shared memory at
// `dst` (1024-byte aligned for 128-byte swizzling), completing the box's
// bytes on `bar` (out-of-bounds elements are filled with zeros and counted).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ uint32_t hmul2_rn(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

}  // namespace coli
