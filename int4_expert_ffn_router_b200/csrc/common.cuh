// common.cuh -- shared definitions of the CUDA path: device weight layout,
// workspace, launch helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/coli_moe.h"

namespace coli {

// ---------------------------------------------------------------------------
// Device-native weight layout (written once by the repack at create).
//
// A matrix of R rows (R % 128 == 0) and C inputs (C % 64 == 0) is stored as
// blocks of 128 rows x one 64-input group:
//     block(rt, g) at ((rt * C/64) + g) * kBlockBytes
// so the 128-row tile `rt` is one contiguous run over its groups. A block is
//     nibbles [8 sub-tiles of 16 rows][4 ti][8 slots][16 bytes]  (4096 B)
//     scales  [8 sub-tiles][8] x {fp16 of row i, fp16 of row i+8} (256 B)
// Lane l = 4*gi + ti of a sub-tile keeps its 16 bytes in slot
// lane_slot(l) = 8 ti + (gi ^ 2 ti) of the sub-tile. Both ways the kernels
// read a sub-tile then touch 8 distinct slots modulo 8 in every quarter-warp
// (conflict-free 16-byte shared-memory loads): a warp reading lanes 0..31
// (quarter-warp q holds gi = 2q, 2q+1 with ti = 0..3), and eight row-owning
// lanes gi = 0..7 reading the slots of one ti. The lane owns rows gi and
// gi+8 and, for each
// 16-input step s = 0..3 of the group, the inputs 16s + {2ti, 2ti+1, 2ti+8,
// 2ti+9}: 32 nibbles in four 32-bit words, word s holding
//     bits 0-3  (row gi,   col 2ti)    bits 16-19 (row gi,   col 2ti+1)
//     bits 4-7  (row gi+8, col 2ti)    bits 20-23 (row gi+8, col 2ti+1)
//     bits 8-11 (row gi,   col 2ti+8)  bits 24-27 (row gi,   col 2ti+9)
//     bits 12-15(row gi+8, col 2ti+8)  bits 28-31 (row gi+8, col 2ti+9)
// as offset-binary codes v = q + 8 in [0, 15]. This is the A-fragment order
// of a 16x16 tensor-core tile, and it lets a CUDA-core lane turn each nibble
// into a float with one logic op (the nibble lands in an fp32 mantissa).
//
// Gate and up are stored as one matrix of 2I rows interleaved by 8: rows
// 16b..16b+7 are gate rows 8b..8b+7 and rows 16b+8..16b+15 are up rows
// 8b..8b+7, so the lane that owns row gi also owns the matching up row gi+8
// and SwiGLU is formed in registers.
// ---------------------------------------------------------------------------
constexpr int kGroup = 64;
constexpr int kTileRows = 128;
// 16-byte slot of lane l = 4*gi + ti within a 512-byte sub-tile.
__host__ __device__ constexpr int lane_slot(int l) { return (l & 3) * 8 + ((l >> 2) ^ (2 * (l & 3))); }
constexpr bool lane_slots_conflict_free() {
    for (int q = 0; q < 4; ++q) {  // a warp reading lanes 0..31, one quarter-warp at a time
        int seen = 0;
        for (int l = 8 * q; l < 8 * q + 8; ++l) seen |= 1 << (lane_slot(l) & 7);
        if (seen != 0xFF) return false;
    }
    for (int ti = 0; ti < 4; ++ti) {  // rows gi = 0..7 reading the slots of one ti
        int seen = 0;
        for (int gi = 0; gi < 8; ++gi) seen |= 1 << (lane_slot(4 * gi + ti) & 7);
        if (seen != 0xFF) return false;
    }
    return true;
}
static_assert(lane_slots_conflict_free(), "every quarter-warp reads 8 distinct 16-byte slots modulo 8");
constexpr int kSubRows = 16;
constexpr int kNibbleBytes = 4096;
constexpr int kScaleBytes = 256;
constexpr int kBlockBytes = kNibbleBytes + kScaleBytes;  // 4352

// CUDA-core expert kernels: tokens per pass over a weight tile (one work item).
constexpr int kCoreTok = 4;
// Tensor-core path: tokens of one expert per GEMM tile (the MMA N).
constexpr int kTcMaxTok = 128;
constexpr int kMaxStages = 24;
// Word of the layer's control block where a persistent kernel that gave up
// on a bounded wait records its site code (0: none); alone in its 128-byte line.
constexpr int kCtlError = 128;
// Code in that word of a decode work item whose positions exceed its operand
// buffer (a broken launch invariant; the item is not staged and the launch stops).
constexpr int kCtlErrBufferOverflow = 13;

inline int64_t matrix_bytes(int rows, int cols) {
    return (int64_t)(rows / kTileRows) * (cols / kGroup) * kBlockBytes;
}

struct Dims {
    int H, I, E, K, S, max_tokens;
    int64_t gu_bytes;      // gate/up matrix [2I][H]
    int64_t d_bytes;       // down matrix [H][I]
    int64_t expert_stride; // gu_bytes + d_bytes (multiple of 256)
    const int32_t* slot_of;  // device [E + S]: weight slot of each expert (expert cache), or NULL: slot = id
};

// Byte offset of expert e's weights in the layer's weight pool.
__device__ __forceinline__ size_t expert_offset(const Dims& d, int e) {
    return (size_t)(d.slot_of ? __ldg(d.slot_of + e) : e) * (size_t)d.expert_stride;
}

// Per-call workspace views (device pointers into the layer's workspace).
struct Plan {
    int32_t* ids;        // [T][K]
    float* w;            // [T][K]
    int32_t* cnt;        // [E]
    int32_t* off;        // [E+1]
    int32_t* unique;     // [E]
    int32_t* n_unique;   // [1]
    int32_t* pos;        // [T][K] -> permuted position
    int32_t* tok;        // [T*K + S*T] permuted token list (shared experts appended)
    int32_t* act_expert; // [E+S] expert id of active slot a (unique experts, then shared)
    int32_t* act_off;    // [E+S] first permuted position of active expert a
    int32_t* act_cnt;    // [E+S] tokens of active expert a
    int32_t* n_active;   // [1] n_unique + S
    int32_t* act_chunk;  // [E+S+1] prefix of ceil(act_cnt / kCoreTok) over the active experts
};

// ---------------------------------------------------------------------------
// Small device helpers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ldg_stream32(const void* p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t orv) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(orv));  // (a & b) | c
    return d;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + __expf(-z)); }
// silu with the approximate division (relative error a few ulp)
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

}  // namespace coli

namespace coli {

// ---------------------------------------------------------------------------
// mbarrier / bulk-copy / ordering helpers (sm_90+ PTX, used on sm_100a).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test of a phase (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may sleep until the phase completes or
// `ns` nanoseconds pass (it is woken when the phase completes), so waiting
// warps do not spend issue slots polling.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bulk copy global -> this CTA's shared memory, completing on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// As bulk_g2s, with an L2 cache policy (createpolicy): data read once, such as
// streamed weights, can be marked to leave L2 first.
__device__ __forceinline__ void bulk_g2s_policy(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                                uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void named_bar(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace coli
