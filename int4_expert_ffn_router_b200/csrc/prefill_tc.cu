// prefill_tc.cu -- the expert FFNs of a token batch on the sm_100a tensor
// cores (tcgen05): per-expert grouped GEMMs over the batch-union plan.
//
// The layer (Colibrì pages: experts are three int4 matrices in 64-input
// groups; every token goes to its top-8 experts plus the shared expert; the
// batch reads each distinct expert once) becomes, per active expert e with
// tokens X_e (rows of the fp16 operand written in position order, so the
// rows of one expert are consecutive):
//     H_e = silu(X_e G_e^T) * (X_e U_e^T)      gate/up GEMM + SwiGLU epilogue
//     y  += w_e * (H_e D_e^T)                   down GEMM + weighted scatter-add
// Each GEMM runs as one persistent kernel: a work item is (token tile of up to
// 128 tokens of one expert) x (two 128-row weight tiles). Per 64-input block:
//   producer thread  bulk-copies the two int4 weight blocks (2 x 4352 B) and
//                    loads the 64-element slices of the tile's token rows (one
//                    TMA tile load from the position-ordered operand) into a
//                    128-byte-swizzled K-major operand in shared memory;
//   transform warps  dequantise one weight row per thread (exact int4 ->
//                    fp16 via the 0x6400 magic, times the fp16 group scale,
//                    one rounding) and store it to tensor memory;
//   MMA thread       issues tcgen05.mma M=128 N=tile K=16 with A from tensor
//                    memory and B from shared memory into two fp32
//                    accumulators in tensor memory;
// and after the last block the transform warps read the accumulators back
// (tcgen05.ld) for the epilogue.
//
// Numerics. Tensor-core operands are fp16: a token row is scaled by a power
// of two so its largest magnitude lies in [2^14, 2^15), which makes the bf16
// -> fp16 conversion exact; the epilogue undoes the scale. The SwiGLU output
// h is stored as fp16 after scaling by a per-token power of two 2^f chosen from
// the bound |h| <= L1(gate row) * L1(up row) * max|x|^2 (the layer's largest
// product of row L1 norms, measured when the weights are loaded), so h cannot
// overflow fp16; the down epilogue multiplies by w / 2^f. Every weight is
// rounded once to fp16 (relative error <= 2^-11); all sums are fp32.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace coli {
namespace {

constexpr int kSStages = 8;                        // shared-memory stages (weights + token slices)
constexpr int kAStages = 2;                        // tensor-memory stages, each two 64-input blocks
constexpr int kBTileBytes = kTcMaxTok * 128;       // token slice: 128 rows x 64 fp16
constexpr int kWStageBytes = 2 * kBlockBytes;      // two 128-row tiles
// Transform warp w = 8 hb + 4 rt2 + q dequantises rows 32q..32q+31 (its
// TMEM lane quarter) of row tile rt2 for block hb of every pair of 64-input
// blocks (so both halves of an A stage are produced in parallel), and in the
// epilogue handles the accumulator columns of chunks 16j..16j+15 with
// j % 2 == hb.
constexpr int kTransformWarps = 16;
constexpr int kProducerWarps = 1;
// Two MMA warps (converged, one elected lane issues): warp kMmaWarp + t2
// drives the accumulator of row tile t2, 8 MMAs (one A stage) per wait.
constexpr int kProducerWarp = kTransformWarps;                     // 16
constexpr int kMmaWarp = kTransformWarps + kProducerWarps;          // 17
constexpr int kThreadsTc = (kMmaWarp + 2) * 32;                     // 608
constexpr uint32_t kTmemCols = 512;
// Tensor memory columns: A stage s (two 64-input blocks of both row tiles)
// at 128 s, + 64 t2 for row tile t2, + 32 hb for block hb of the pair (16
// fp16 of K per MMA = 8 columns); the two fp32 accumulators from column 256
// (kTcMaxTok columns each).
constexpr int kABase = 0;
constexpr int kAccBase = kAStages * 128;           // 256
constexpr int kAccCols = kTcMaxTok;                // accumulator of one row tile
static_assert(kAccBase + 2 * kAccCols <= (int)kTmemCols, "tensor memory budget");
constexpr uint64_t kTcWaitNs = 1000000000ull;      // every wait gives up after 1 s (default)

// shared memory map (offsets from a 1024-aligned base)
constexpr int kOffB = 0;
constexpr int kOffW = kOffB + kSStages * kBTileBytes;
constexpr int kOffSlot = kOffW + kSStages * kWStageBytes;          // per transform warp: its columns' factors
constexpr int kSlotPerWarp = kTcMaxTok / 2;
constexpr int kOffBar = kOffSlot + kTransformWarps * kSlotPerWarp * 16;
constexpr int kNumBars = 2 * kSStages + 4 * kAStages + 6;
static_assert(kSStages % 2 == 0, "a pair of blocks never wraps the shared-memory ring");
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemTc = kOffMisc + 16 + 1024;                      // + alignment slack
static_assert(kOffBar % 8 == 0, "alignment");
constexpr int kSmallBox = 32;                      // token rows per TMA load for tiles of up to 32 tokens

struct __align__(64) TcArgs {
    CUtensorMap tmap_big;   // 2D map over the token operand (xs or h16), box 64 x kTcMaxTok rows
    CUtensorMap tmap_small; // the same with box 64 x kSmallBox rows (tiles of up to kSmallBox tokens)
    const uint8_t* weights;
    int64_t expert_stride;
    const int32_t* slot_of;   // expert -> weight slot (expert cache) or NULL
    int64_t mat_offset;     // 0 (gate/up) or the down matrix offset within an expert
    int KB;                 // 64-input blocks per row (H/64 or I/64)
    int RT2;                // pairs of 128-row tiles
    const float4* slot;     // per position {x scale, h scale, w / h scale, token}
    const int4* tiles;      // {weight index, first position, tokens, 0}
    const int* n_tiles;
    __half* h16;            // gate/up output [slots][I]
    float* y32;             // down output [T][H] (accumulated)
    int I, H;
    int* err;               // timeout site (control block)
    uint64_t wait_ns;       // bound of every wait
    int wait_test;          // testing aid: MMA warp 0 first waits on a barrier that nothing completes
    long long* trace;       // CTA 0 timeline (clock64 stamps) or NULL
    int trace_cap;          // 64-input blocks recorded
};

// Timeline of CTA 0 (when a.trace is set): per 64-input block `it`,
// trace[it * 8 + j] for j = 0 transform warp 0 has the block, 1 its A
// stage is free, 2 its stores are issued, 3 MMA has the block, 4 MMA has the
// A stage, 5 MMAs issued, 6 producer has the stage, 7 copies issued; then per
// item i, trace[cap * 8 + 2 i] epilogue start, [.. + 1] epilogue end.
// Recorded only in profiling builds (COLI_TC_TRACE=1): the stamps cost
// issue slots in the loops they time.
#ifndef COLI_TC_TRACE
#define COLI_TC_TRACE 0
#endif
__device__ __forceinline__ void tc_stamp(const TcArgs& a, uint32_t it, int j) {
    if constexpr (COLI_TC_TRACE != 0) {
        if (a.trace && blockIdx.x == 0 && it < (uint32_t)a.trace_cap) a.trace[(size_t)it * 8 + j] = clock64();
    }
}
__device__ __forceinline__ void tc_stamp_item(const TcArgs& a, uint32_t i, int j) {
    if constexpr (COLI_TC_TRACE != 0) {
        if (a.trace && blockIdx.x == 0 && i < 64u) a.trace[(size_t)a.trace_cap * 8 + 2 * i + j] = clock64();
    }
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int site,
                                        uint64_t limit);

// Every lane polls (a one-lane poll plus broadcast costs more); the warp goes
// on only if all lanes saw the phase complete, so warp-collective tcgen05
// instructions stay converged.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err,
                                             int site, uint64_t limit) {
    const bool ok = tc_wait(bar, parity, abort_flag, err, site, limit);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int site,
                                        uint64_t limit) {
    // sleep in the barrier for up to 0.2 ms at a time; the bound stays 1 s
    if (mbar_try_wait_sleep(bar, parity, 200000)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 200000)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit) {
            *abort_flag = 1;
            atomicCAS(err, 0, site);
            return false;
        }
    }
}

// kPairs (gate/up only): the token operand holds two fp16 rows per position,
// hi and lo parts of an fp32 input; the MMA columns 2i and 2i+1 of a tile are
// the two parts of its token i and the epilogue adds them.
template <int kPhase, bool kPairs>
__global__ void __launch_bounds__(kThreadsTc, 1) moe_prefill_tc_kernel(const __grid_constant__ TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint64_t* full = bars;                        // [kSStages] producer -> transform (1 arrival + bytes)
    uint64_t* sempty = full + kSStages;           // [kSStages] both MMA issuers -> producer
    uint64_t* aready = sempty + kSStages;         // [kAStages][2] transform warps of tile t2 -> issuer t2
    uint64_t* aempty = aready + 2 * kAStages;     // [kAStages][2] issuer t2 -> transform warps of tile t2
    uint64_t* accfull = aempty + 2 * kAStages;    // [2] issuer t2 -> epilogue of tile t2
    uint64_t* accempty = accfull + 2;             // [2] epilogue of tile t2 -> issuer t2
    uint64_t* drained = accempty + 2;             // [2] issuer t2: all its MMAs complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&sempty[s], 2);
        }
        for (int s = 0; s < 2 * kAStages; ++s) {
            mbar_init(&aready[s], kTransformWarps / 2);  // 4 quarters x 2 blocks of the pair
            mbar_init(&aempty[s], 1);
        }
        for (int t2 = 0; t2 < 2; ++t2) {
            mbar_init(&accfull[t2], 1);
            mbar_init(&accempty[t2], kTransformWarps / 2);
            mbar_init(&drained[t2], 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) {
        tc_alloc(tmem_slot, kTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int n_items = *a.n_tiles * a.RT2;
    const int KB = a.KB;

    if (warp < kTransformWarps) {
        // ------------------------------------------------ transform + epilogue
        const int q = warp & 3, rt2 = (warp >> 2) & 1, hb = warp >> 3, kh = hb;
        const int m = 32 * q + lane;                 // row within the 128-row tile
        const int sub = m >> 4, gi = m & 7, isb = (m >> 3) & 1;
        const uint32_t mask = isb ? 0x00F000F0u : 0x000F000Fu;
        const uint32_t mul = isb ? 0x2C002C00u : 0x3C003C00u;   // 1/16 : 1
        const uint32_t add = isb ? 0xD480D480u : 0xE408E408u;   // -72 : -1032
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        // factors of this warp's columns: local index (j / 2) * 16 + (c & 15) for column c of chunk j
        float4* sinfo = reinterpret_cast<float4*>(sm + kOffSlot) + warp * kSlotPerWarp;
        uint32_t it0 = 0, icount = 0;  // block counter at the item's first block (KB is even)
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x, it0 += KB) {
            const int4 tile = a.tiles[item / a.RT2];
            const int pair = item % a.RT2;
            const int n = tile.z, start = tile.y;
            const int ncol = kPairs ? 2 * n : n, nm = (ncol + 15) & ~15;  // MMA columns
            constexpr int kTokPerChunk = kPairs ? 8 : 16;                    // tokens per 16 columns
#pragma unroll
            for (int h = 0; h < kSlotPerWarp / 32; ++h) {
                const int lc = lane + 32 * h;  // local index (j / 2) * kTokPerChunk + i for token i of chunk j
                const int c = kTokPerChunk * (2 * (lc / kTokPerChunk) + kh) + (lc % kTokPerChunk);
                if (c < n && lc < (kSlotPerWarp / 16) * kTokPerChunk) sinfo[lc] = a.slot[start + c];
            }
            // phases of this warp's next block seen complete while it worked on the current one
            bool seen_full = false, seen_aempty = false;
            for (int kb = hb; kb < KB; kb += 2) {
                const uint32_t it = it0 + kb;
                const uint32_t p2 = it >> 1;           // A stage use counter
                const uint32_t s = it % kSStages, sa = p2 % kAStages;
                if (!seen_full && !tc_wait_warp(&full[s], (it / kSStages) & 1, abort_flag, a.err, 21, a.wait_ns)) { ok = false; break; }
                if (warp == 0 && lane == 0) tc_stamp(a, it, 0);
                if (!seen_aempty && !tc_wait_warp(&aempty[2 * sa + rt2], ((p2 / kAStages) & 1) ^ 1, abort_flag, a.err, 22, a.wait_ns)) { ok = false; break; }
                if (warp == 0 && lane == 0) tc_stamp(a, it, 1);
                tc_fence_after();
                const uint8_t* blk = sm + kOffW + s * kWStageBytes + rt2 * kBlockBytes;
                const uint8_t* subp = blk + sub * 512;  // lane 4gi+ti of the sub-tile at lane_slot(4gi+ti)
                uint4 wv[4];
#pragma unroll
                for (int ti = 0; ti < 4; ++ti) wv[ti] = *reinterpret_cast<const uint4*>(subp + 16 * lane_slot(4 * gi + ti));
                const uint32_t sp = *reinterpret_cast<const uint32_t*>(blk + kNibbleBytes + sub * 32 + gi * 4);
                // test the next block's phases now (non-blocking): the answers are read after the
                // dequantisation, so a barrier that is already complete costs no wait latency
                bool nf = false, na = false;
                if (kb + 2 < KB) {
                    const uint32_t itn = it + 2, p2n = itn >> 1;
                    nf = mbar_test_wait(&full[itn % kSStages], (itn / kSStages) & 1);
                    na = mbar_test_wait(&aempty[2 * (p2n % kAStages) + rt2], ((p2n / kAStages) & 1) ^ 1);
                }
                const uint32_t s2 = __byte_perm(sp, 0, isb ? 0x3232 : 0x1010);
                uint32_t r[32];
#pragma unroll
                for (int ti = 0; ti < 4; ++ti) {
                    const uint32_t words[4] = {wv[ti].x, wv[ti].y, wv[ti].z, wv[ti].w};
#pragma unroll
                    for (int ws = 0; ws < 4; ++ws) {
                        const uint32_t w = words[ws];
                        const uint32_t lo = hfma2_u(lop3_and_or(w, mask, 0x64006400u), mul, add);
                        const uint32_t hi = hfma2_u(lop3_and_or(w >> 8, mask, 0x64006400u), mul, add);
                        r[8 * ws + ti] = hmul2_rn(lo, s2);      // inputs 16ws + 2ti, +1
                        r[8 * ws + 4 + ti] = hmul2_rn(hi, s2);  // inputs 16ws + 2ti + 8, +9
                    }
                }
                const uint32_t ta = tmem + lane_base + kABase + 128 * sa + 64 * rt2 + 32 * hb;
                tc_st16(ta, r);
                tc_st16(ta + 16, r + 16);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                mbar_arrive_elect(&aready[2 * sa + rt2]);
                if (warp == 0 && lane == 0) tc_stamp(a, it, 2);
                seen_full = __all_sync(0xffffffffu, nf);
                seen_aempty = __all_sync(0xffffffffu, na);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (!tc_wait_warp(&accfull[rt2], icount & 1, abort_flag, a.err, 23, a.wait_ns)) { ok = false; break; }
            if (warp == 0 && lane == 0) tc_stamp_item(a, icount, 0);
            tc_fence_after();
            const uint32_t tacc = tmem + lane_base + kAccBase + rt2 * kAccCols;
            const int row = (2 * pair + rt2) * 128 + m;  // row of the weight matrix
            for (int j = kh; 16 * j < nm; j += 2) {
                const int c16 = 16 * j, lc0 = (j >> 1) * 16;
                uint32_t v[16];
                tc_ld16_wait(tacc + c16, v);
                if (kPhase == 0 && kPairs) {
                    // columns 2i, 2i+1: hi and lo parts of token c16/2 + i. The gate lane (isb = 0)
                    // forms h for tokens 0..3 of the chunk, the up lane (isb = 1) for 4..7.
                    const int jh = (row >> 4) * 8 + (row & 7);
                    float tv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) tv[i] = __uint_as_float(v[2 * i]) + __uint_as_float(v[2 * i + 1]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float send = isb ? tv[i] : tv[4 + i];
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
                        const float g = isb ? recv : tv[i];
                        const float u = isb ? tv[4 + i] : recv;
                        const int ti = 4 * isb + i;          // token within the chunk
                        const int nn = c16 / 2 + ti;
                        if (nn < n) {
                            const float4 si = sinfo[(j >> 1) * 8 + ti];
                            const float hv = silu_fast(g * si.x) * (u * si.x);
                            a.h16[(size_t)(start + nn) * a.I + jh] = __float2half_rn(hv * si.y);
                        }
                    }
                } else if (kPhase == 0) {
                    // gate row (isb = 0) and up row (isb = 1) of the same h index sit 8 lanes apart:
                    // the gate lane forms h for even tokens, the up lane for odd ones.
                    const int jh = (row >> 4) * 8 + (row & 7);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float send = __uint_as_float(isb ? v[2 * i] : v[2 * i + 1]);
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
                        const float g = isb ? recv : __uint_as_float(v[2 * i]);
                        const float u = isb ? __uint_as_float(v[2 * i + 1]) : recv;
                        const int nn = c16 + 2 * i + isb;
                        if (nn < n) {
                            const float4 si = sinfo[lc0 + 2 * i + isb];
                            const float hv = silu_fast(g * si.x) * (u * si.x);
                            a.h16[(size_t)(start + nn) * a.I + jh] = __float2half_rn(hv * si.y);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int nn = c16 + i;
                        if (nn < n) {
                            const float4 si = sinfo[lc0 + i];
                            const int t = __float_as_int(si.w);
                            atomicAdd(a.y32 + (size_t)t * a.H + row, __uint_as_float(v[i]) * si.z);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            mbar_arrive_elect(&accempty[rt2]);
            if (warp == 0 && lane == 0) tc_stamp_item(a, icount, 1);
            ++icount;
        }
    } else if (warp == kProducerWarp) {
      if (lane == 0) {
        // ------------------------------------------------------- producer
        // Per block: the two weight blocks (bulk copies) and the tile's token
        // rows start..start+n-1 of the position-ordered operand (one TMA
        // tile load; rows past the tile belong to other experts or lie past
        // the tensor, where TMA fills zeros; their columns are never read).
        uint32_t it = 0;
        bool ok = true;
        const uint64_t wpolicy = l2_policy_evict_first();
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int4 tile = a.tiles[item / a.RT2];
            const int pair = item % a.RT2;
            const int n = tile.z, start = tile.y;
            const int rows = kPairs ? 2 * n : n, row0 = kPairs ? 2 * start : start;
            const bool small = rows <= kSmallBox;
            const void* map = small ? (const void*)&a.tmap_small : (const void*)&a.tmap_big;
            const uint32_t tx_bytes = 2 * kBlockBytes + (small ? kSmallBox : kTcMaxTok) * 128;
            const size_t eslot = a.slot_of ? (size_t)__ldg(a.slot_of + tile.x) : (size_t)tile.x;
            const uint8_t* w0 = a.weights + eslot * a.expert_stride + a.mat_offset +
                                (size_t)(2 * pair) * KB * kBlockBytes;
            const uint8_t* w1 = w0 + (size_t)KB * kBlockBytes;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const uint32_t s = it % kSStages;
                if (!tc_wait(&sempty[s], ((it / kSStages) & 1) ^ 1, abort_flag, a.err, 24, a.wait_ns)) { ok = false; break; }
                tc_stamp(a, it, 6);
                uint8_t* wdst = sm + kOffW + s * kWStageBytes;
                mbar_arrive_expect_tx(&full[s], tx_bytes);
                // weights leave L2 first, so the tile's token rows (read again by every pair of row
                // tiles) stay there
                bulk_g2s_policy(wdst, w0 + (size_t)kb * kBlockBytes, kBlockBytes, &full[s], wpolicy);
                bulk_g2s_policy(wdst + kBlockBytes, w1 + (size_t)kb * kBlockBytes, kBlockBytes, &full[s], wpolicy);
                tma_load_2d(smem_addr(sm + kOffB + s * kBTileBytes), map, kb * 64, row0, &full[s]);
                tc_stamp(a, it, 7);
            }
        }
        // copies still in flight (after an abort) must land before the CTA exits
        const uint32_t first = it > (uint32_t)kSStages ? it - kSStages : 0;
        const uint64_t t0 = globaltimer_ns();
        for (uint32_t k = first; k < it; ++k) {
            while (!mbar_try_wait(&full[k % kSStages], (k / kSStages) & 1) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
      }
      __syncwarp();
    } else {
        // ------------------------------------------------------------ MMA
        // issuer warp t2 (converged; one elected lane issues): accumulator of
        // row tile t2, A from its half of each A stage
        const int t2 = warp - kMmaWarp;
        const uint32_t dacc = tmem + kAccBase + t2 * kAccCols;
        const uint32_t abase = tmem + kABase + 64 * t2;
        const uint64_t bdesc0 = tc_sdesc_sw128(smem_addr(sm + kOffB));
        uint32_t it = 0, icount = 0;
        bool ok = true, issued = false;
        // testing aid: drained[0] completes only after this warp's own final commit, so the launch gives up
        if (a.wait_test && t2 == 0) ok = tc_wait_warp(&drained[0], 0, abort_flag, a.err, 29, a.wait_ns);
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int4 tile = a.tiles[item / a.RT2];
            const int nm = ((kPairs ? 2 * tile.z : tile.z) + 15) & ~15;
            const uint32_t idesc = tc_idesc_f16(nm, false);
            if (!tc_wait_warp(&accempty[t2], (icount & 1) ^ 1, abort_flag, a.err, 25, a.wait_ns)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < KB; kb += 2, it += 2) {
                const uint32_t p2 = it >> 1;
                const uint32_t s0 = it % kSStages, sa = p2 % kAStages;
                // aready implies full: the transform warps waited for both blocks' stages before arriving
                if (!tc_wait_warp(&aready[2 * sa + t2], (p2 / kAStages) & 1, abort_flag, a.err, 27, a.wait_ns)) { ok = false; break; }
                tc_fence_after();
                const uint64_t bd0 = bdesc0 + s0 * (kBTileBytes >> 4);
                const uint64_t bd1 = bdesc0 + ((s0 + 1) % kSStages) * (kBTileBytes >> 4);
                const uint32_t acol = abase + 128 * sa;
                tc_mma8_commit3(dacc, acol, bd0, bd1, idesc, kb != 0, smem_addr(&sempty[s0]),
                                smem_addr(&sempty[(s0 + 1) % kSStages]), smem_addr(&aempty[2 * sa + t2]));
                issued = true;
                if (t2 == 0 && lane == 0) {
                    tc_stamp(a, it, 5);
                    tc_stamp(a, it + 1, 5);
                }
            }
            if (!ok) break;
            tc_commit_elect(&accfull[t2]);
            ++icount;
        }
        if (issued) {
            // every MMA must complete before the tensor memory is released
            tc_commit_elect(&drained[t2]);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&drained[t2], 0) && globaltimer_ns() - t0 < a.wait_ns) {
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tc_dealloc(tmem, kTmemCols);
}

// One warp per token: max |x_t|, the power-of-two scales, and the row
// fp16(x_t * 2^e_t) written to every position of the token (its K routed
// positions pos[t][k], then T*K + j*T + t for each shared expert j), so each
// expert's tokens are consecutive rows of xs. bf16 input: one row per
// position (exact). fp32 input: two rows per position, 2p = hi = fp16(x 2^e)
// and 2p+1 = lo = fp16(x 2^e - hi), about 22 significant bits together.
template <typename XT>
__global__ void prefill_prep_kernel(const XT* __restrict__ x, int T, int H, int K, int S,
                                    const int32_t* __restrict__ pos, const float* __restrict__ meta,
                                    __half* __restrict__ xs, float4* __restrict__ tscale) {
    constexpr bool kF32 = sizeof(XT) == 4;
    constexpr int kV = 8;  // elements per lane per step (16 bytes of bf16, 32 of fp32)
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const double bound = (double)meta[0] * (1.0 + 1e-3);  // max_j L1(gate_j) L1(up_j), with rounding margin
    auto load8 = [&](const XT* p, float v[kV]) {
        if constexpr (kF32) {
            const float4 a0 = reinterpret_cast<const float4*>(p)[0], a1 = reinterpret_cast<const float4*>(p)[1];
            v[0] = a0.x; v[1] = a0.y; v[2] = a0.z; v[3] = a0.w; v[4] = a1.x; v[5] = a1.y; v[6] = a1.z; v[7] = a1.w;
        } else {
            const uint4 u = *reinterpret_cast<const uint4*>(p);
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[2 * k] = __uint_as_float(w[k] << 16);
                v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
            }
        }
    };
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
        const XT* row = x + (size_t)t * H;
        float mx = 0.0f;
        for (int i = lane * kV; i < H; i += 32 * kV) {
            float v[kV];
            load8(row + i, v);
#pragma unroll
            for (int k = 0; k < kV; ++k) mx = fmaxf(mx, fabsf(v[k]));
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0, f = 0;
        if (mx > 0.0f && mx <= 3.0e38f) {
            e = min(120, max(-120, 14 - ilogbf(mx)));
            const double hb = bound * (double)mx * (double)mx;
            if (hb > 0.0) f = min(120, max(-120, ilogb(16384.0 / hb)));
        }
        // positions of this token (K <= 32 routed, then S <= 64 shared): position q is held
        // by lane q % 32 in dst_r[q / 32] and broadcast with a shuffle
        const int np = K + S;
        auto position = [&](int q) { return q < K ? pos[(size_t)t * K + q] : T * K + (q - K) * T + t; };
        int dst_r[3];
#pragma unroll
        for (int r = 0; r < 3; ++r) dst_r[r] = 32 * r + lane < np ? position(32 * r + lane) : -1;
        for (int i = lane * kV; i < H; i += 32 * kV) {
            float v[kV];
            load8(row + i, v);
            uint32_t hi4[4], lo4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float a0 = ldexpf(v[2 * k], e), a1 = ldexpf(v[2 * k + 1], e);
                const __half h0 = __float2half_rn(a0), h1 = __float2half_rn(a1);
                hi4[k] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
                if constexpr (kF32) {
                    const __half l0 = __float2half_rn(a0 - __half2float(h0)), l1 = __float2half_rn(a1 - __half2float(h1));
                    lo4[k] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
                }
            }
            const uint4 hv = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
            for (int q = 0; q < np; ++q) {
                const int d = __shfl_sync(0xffffffffu, q < 32 ? dst_r[0] : q < 64 ? dst_r[1] : dst_r[2], q & 31);
                if (d < 0) continue;  // an empty slot (expert of another rank)
                if constexpr (kF32) {
                    reinterpret_cast<uint4*>(xs + (size_t)(2 * d) * H + i)[0] = hv;
                    reinterpret_cast<uint4*>(xs + (size_t)(2 * d + 1) * H + i)[0] =
                        make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
                } else {
                    reinterpret_cast<uint4*>(xs + (size_t)d * H + i)[0] = hv;
                }
            }
        }
        if (lane == 0) tscale[t] = make_float4(ldexpf(1.0f, -e), ldexpf(1.0f, f), ldexpf(1.0f, -f), 0.0f);
    }
}

// Per-position epilogue factors (every CTA, grid-stride) and the tile list
// (CTA 0). Tiles hold at most kTcMaxTok tokens of one expert and are ordered
// by decreasing size.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(Plan p, int T, int K, int S, int max_tok,
                                                            const float4* __restrict__ tscale,
                                                            float4* __restrict__ slot, int4* __restrict__ tiles,
                                                            int* __restrict__ n_tiles) {
    __shared__ int bcnt[kTcMaxTok / 16], bbase[kTcMaxTok / 16], bcur[kTcMaxTok / 16];
    constexpr int NB = kTcMaxTok / 16;
    const int TK = T * K;
    const int stride = gridDim.x * blockDim.x, i0 = blockIdx.x * blockDim.x + threadIdx.x;
    for (int i = i0; i < TK; i += stride) {
        const int t = i / K;
        const float4 ts = tscale[t];
        if (p.pos[i] >= 0) slot[p.pos[i]] = make_float4(ts.x, ts.y, p.w[i] * ts.z, __int_as_float(t));
    }
    for (int i = i0; i < S * T; i += stride) {
        const int t = i % T;
        const float4 ts = tscale[t];
        slot[TK + i] = make_float4(ts.x, ts.y, ts.z, __int_as_float(t));
    }
    if (blockIdx.x != 0) return;
    if (threadIdx.x < NB) bcnt[threadIdx.x] = bcur[threadIdx.x] = 0;
    __syncthreads();
    const int na = *p.n_active;
    for (int pass = 0; pass < 2; ++pass) {
        for (int u = threadIdx.x; u < na; u += blockDim.x) {
            const int cnt = p.act_cnt[u];
            if (cnt <= 0) continue;
            const int nt = (cnt + max_tok - 1) / max_tok;
            const int sz = (cnt + nt - 1) / nt;
            for (int j = 0; j < nt; ++j) {
                const int n = min(sz, cnt - j * sz);
                if (n <= 0) break;
                const int b = (n + 15) / 16 - 1;
                if (pass == 0) {
                    atomicAdd(&bcnt[b], 1);
                } else {
                    const int idx = bbase[b] + atomicAdd(&bcur[b], 1);
                    tiles[idx] = make_int4(p.act_expert[u], p.act_off[u] + j * sz, n, 0);
                }
            }
        }
        __syncthreads();
        if (pass == 0 && threadIdx.x == 0) {
            int run = 0;
            for (int b = NB - 1; b >= 0; --b) {
                bbase[b] = run;
                run += bcnt[b];
            }
            *n_tiles = run;
        }
        __syncthreads();
    }
}

template <typename YT>
__global__ void prefill_out_kernel(const float* __restrict__ y32, const float* __restrict__ residual, size_t n,
                                   YT* __restrict__ y) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x) {
        float4 v = reinterpret_cast<const float4*>(y32)[i];
        if (residual) {
            const float4 r = reinterpret_cast<const float4*>(residual)[i];
            v.x += r.x; v.y += r.y; v.z += r.z; v.w += r.w;
        }
        if constexpr (sizeof(YT) == 4) {
            reinterpret_cast<float4*>(y)[i] = v;
        } else {
            __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
            uint2 o;
            o.x = *reinterpret_cast<uint32_t*>(&lo);
            o.y = *reinterpret_cast<uint32_t*>(&hi);
            reinterpret_cast<uint2*>(y)[i] = o;
        }
    }
}

// One warp per gate/up row pair j: L1 norms of gate row j and up row j from
// the canonical container (two's-complement nibbles, fp16 scales), their
// product folded into meta[0] (max), and max |scale| of the rows into meta[1].
__global__ void l1_bound_kernel(const uint8_t* __restrict__ qg, const uint16_t* __restrict__ sg,
                                const uint8_t* __restrict__ qu, const uint16_t* __restrict__ su, int I, int H,
                                unsigned* __restrict__ meta) {
    const int lane = threadIdx.x & 31;
    const int G = H / 64;
    for (int j = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); j < I; j += gridDim.x * (blockDim.x >> 5)) {
        float l1[2] = {0.0f, 0.0f}, smax = 0.0f;
        for (int mtx = 0; mtx < 2; ++mtx) {
            const uint8_t* qrow = (mtx ? qu : qg) + (size_t)j * (H / 2);
            const uint16_t* srow = (mtx ? su : sg) + (size_t)j * G;
            for (int g = lane; g < G; g += 32) {
                const float s = fabsf(__half2float(__ushort_as_half(srow[g])));
                const uint4* qv = reinterpret_cast<const uint4*>(qrow + g * 32);
                int acc = 0;
                for (int h = 0; h < 2; ++h) {
                    const uint4 v = qv[h];
                    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
                    for (int k = 0; k < 4; ++k)
                        for (int b = 0; b < 8; ++b) {
                            const int c = (int)((words[k] >> (4 * b)) & 0xFu);
                            acc += c >= 8 ? 16 - c : c;  // |two's-complement nibble|
                        }
                }
                l1[mtx] += (float)acc * s;
                smax = fmaxf(smax, s);
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            l1[0] += __shfl_xor_sync(0xffffffffu, l1[0], o);
            l1[1] += __shfl_xor_sync(0xffffffffu, l1[1], o);
            smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
        }
        if (lane == 0) {
            atomicMax(&meta[0], __float_as_uint(l1[0] * l1[1]));  // non-negative floats order as integers
            atomicMax(&meta[1], __float_as_uint(smax));
        }
    }
}

// max |scale| of a canonical scale array (down matrix) into meta[1].
__global__ void scale_max_kernel(const uint16_t* __restrict__ s, size_t n, unsigned* __restrict__ meta) {
    float m = 0.0f;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(__half2float(__ushort_as_half(s[i]))));
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((threadIdx.x & 31) == 0) atomicMax(&meta[1], __float_as_uint(m));
}

}  // namespace

size_t prefill_tc_smem_bytes() { return kSmemTc; }

// 2D fp16 tensor map over rows x cols (row pitch cols * 2 bytes) for the
// token operand: box 64 elements x box_rows rows, 128-byte swizzle.
cudaError_t make_token_map(void* map, const void* base, int rows, int cols, int box_rows) {
    using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<EncodeFn>(fn);
    }
    if (((uintptr_t)base & 15u) || (cols * 2) % 16 || rows < 1 || box_rows < 1 || box_rows > 256)
        return cudaErrorInvalidValue;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = encode(reinterpret_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                              const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int prefill_tc_max_tiles(const Dims& d, int T) {
    return d.E + d.S + (T * d.K + d.S * T) / kTcMaxTok + 1;
}

cudaError_t launch_l1_bound(const uint8_t* q, const uint16_t* s, int H, int I, unsigned* meta, cudaStream_t st) {
    const size_t mq = (size_t)I * H / 2, ms = (size_t)I * H / 64;
    l1_bound_kernel<<<256, 256, 0, st>>>(q, s, q + mq, s + ms, I, H, meta);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    scale_max_kernel<<<256, 256, 0, st>>>(s + 2 * ms, ms, meta);
    return cudaGetLastError();
}

cudaError_t launch_prefill_prep(const void* x, coli_dtype dt, int T, int H, int K, int S, const int32_t* pos,
                                const float* meta, __half* xs, float4* tscale, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int grid = (T + 7) / 8 < 1184 ? (T + 7) / 8 : 1184;
    if (dt == COLI_F32)
        prefill_prep_kernel<float><<<grid, 256, 0, st>>>((const float*)x, T, H, K, S, pos, meta, xs, tscale);
    else
        prefill_prep_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, T, H, K, S, pos, meta, xs,
                                                                 tscale);
    return cudaGetLastError();
}

cudaError_t launch_prefill_plan(const Plan& p, int T, int K, int S, int max_tok, const float4* tscale, float4* slot,
                                int4* tiles, int* n_tiles, cudaStream_t st) {
    const int positions = T * K + S * T;
    const int grid = std::max(1, std::min(148, (positions + 1023) / 1024));
    prefill_plan_kernel<<<grid, 1024, 0, st>>>(p, T, K, S, max_tok, tscale, slot, tiles, n_tiles);
    return cudaGetLastError();
}

cudaError_t launch_prefill_gemm(int phase, bool pairs, const uint8_t* weights, const Dims& d, const void* token_maps,
                                const Plan& p, const float4* slot, const int4* tiles, const int* n_tiles, __half* h16,
                                float* y32, int* err, int n_sm, long long* trace, int trace_cap, int64_t wait_ns,
                                int wait_test, cudaStream_t st) {
    TcArgs a;
    memcpy(&a.tmap_big, token_maps, sizeof(CUtensorMap));
    memcpy(&a.tmap_small, static_cast<const uint8_t*>(token_maps) + sizeof(CUtensorMap), sizeof(CUtensorMap));
    a.trace = trace;
    a.trace_cap = trace_cap;
    a.weights = weights;
    a.expert_stride = d.expert_stride;
    a.slot_of = d.slot_of;
    a.mat_offset = phase == 0 ? 0 : d.gu_bytes;
    a.KB = phase == 0 ? d.H / kGroup : d.I / kGroup;
    a.RT2 = phase == 0 ? (2 * d.I / kTileRows) / 2 : (d.H / kTileRows) / 2;
    a.slot = slot;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.h16 = h16;
    a.y32 = y32;
    a.I = d.I;
    a.H = d.H;
    a.err = err;
    a.wait_ns = wait_ns > 0 ? (uint64_t)wait_ns : kTcWaitNs;
    a.wait_test = wait_test;
    cudaError_t e;
    auto run = [&](auto kern) {
        cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
        if (r != cudaSuccess) return r;
        kern<<<n_sm, kThreadsTc, kSmemTc, st>>>(a);
        return cudaSuccess;
    };
    if (phase == 0)
        e = pairs ? run(moe_prefill_tc_kernel<0, true>) : run(moe_prefill_tc_kernel<0, false>);
    else
        e = run(moe_prefill_tc_kernel<1, false>);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_prefill_out(const float* y32, const float* residual, int T, int H, void* y, coli_dtype dt,
                               cudaStream_t st) {
    const size_t n = (size_t)T * H;
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n / 4 + 255) / 256;
    const int grid = (int)(blocks < 4736 ? blocks : 4736);
    if (dt == COLI_F32)
        prefill_out_kernel<float><<<grid, 256, 0, st>>>(y32, residual, n, (float*)y);
    else
        prefill_out_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(y32, residual, n, (__nv_bfloat16*)y);
    return cudaGetLastError();
}

}  // namespace coli
