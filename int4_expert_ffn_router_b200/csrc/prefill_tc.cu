// prefill_tc.cu -- the expert FFNs of a token batch on the sm_100a tensor
// cores (tcgen05): per-expert grouped GEMMs over the batch-union plan.
//
// The layer (Colibrì pages: experts are three int4 matrices in 64-input
// groups; every token goes to its top-8 experts plus the shared expert; the
// batch reads each distinct expert once) becomes, per active expert e with
// tokens X_e (gathered by index, never copied out):
//     H_e = silu(X_e G_e^T) * (X_e U_e^T)      gate/up GEMM + SwiGLU epilogue
//     y  += w_e * (H_e D_e^T)                   down GEMM + weighted scatter-add
// Each GEMM runs as one persistent kernel: a work item is (token tile of up to
// 128 tokens of one expert) x (two 128-row weight tiles). Per 64-input block:
//   producer warps   bulk-copy the two int4 weight blocks (2 x 4352 B) and
//                    gather the 64-element slices of the tile's token rows into
//                    a 128-byte-swizzled K-major operand in shared memory;
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
#include "common.cuh"
#include "int4_mma.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"

namespace coli {
namespace {

constexpr int kSStages = 6;                        // shared-memory stages (weights + token slices)
constexpr int kAStages = 4;                        // tensor-memory stages of dequantised weights
constexpr int kBTileBytes = kTcMaxTok * 128;       // token slice: 128 rows x 64 fp16
constexpr int kWStageBytes = 2 * kBlockBytes;      // two 128-row tiles
constexpr int kTransformWarps = 8;
constexpr int kProducerThreads = 64;
constexpr int kMmaWarp = kTransformWarps + kProducerThreads / 32;  // 10
constexpr int kThreadsTc = (kMmaWarp + 1) * 32;                     // 352
constexpr uint32_t kTmemCols = 512;
// Tensor memory columns: dequantised weights of A stage s at 64 s (+32 for
// the second row tile; 16 fp16 of K per MMA = 8 columns), the two fp32
// accumulators from column 256 (kTcMaxTok columns each).
constexpr int kABase = 0;
constexpr int kAccBase = kAStages * 64;            // 256
constexpr int kAccCols = kTcMaxTok;                // accumulator of one row tile
static_assert(kAccBase + 2 * kAccCols <= (int)kTmemCols, "tensor memory budget");
constexpr uint64_t kTcWaitNs = 1000000000ull;      // every wait gives up after 1 s

// shared memory map (offsets from a 1024-aligned base)
constexpr int kOffB = 0;
constexpr int kOffW = kOffB + kSStages * kBTileBytes;
constexpr int kOffBar = kOffW + kSStages * kWStageBytes;
constexpr int kNumBars = 2 * kSStages + 2 * kAStages + 3;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemTc = kOffMisc + 16 + 1024;                      // + alignment slack
static_assert(kOffBar % 8 == 0, "alignment");
static_assert(kTcMaxTok % (kProducerThreads / 8) == 0, "producer row split");

struct TcArgs {
    const uint8_t* weights;
    int64_t expert_stride;
    int64_t mat_offset;     // 0 (gate/up) or the down matrix offset within an expert
    int KB;                 // 64-input blocks per row (H/64 or I/64)
    int RT2;                // pairs of 128-row tiles
    const __half* src;      // gate/up: x16 [T][H]; down: h16 [slots][I]
    int src_pitch;          // elements per source row
    const int32_t* tok;     // gate/up: token of each position
    const float4* slot;     // per position {x scale, h scale, w / h scale, token}
    const int4* tiles;      // {weight index, first position, tokens, 0}
    const int* n_tiles;
    __half* h16;            // gate/up output [slots][I]
    float* y32;             // down output [T][H] (accumulated)
    int I, H;
    int* err;               // timeout site (control block)
};

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int site);

// All lanes of a warp wait; the warp goes on only if every lane saw the phase
// complete, so warp-collective tcgen05 instructions stay converged.
__device__ __forceinline__ bool tc_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err,
                                             int site) {
    const bool ok = tc_wait(bar, parity, abort_flag, err, site);
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int site) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kTcWaitNs) {
            *abort_flag = 1;
            atomicCAS(err, 0, site);
            return false;
        }
    }
}

template <int kPhase>
__global__ void __launch_bounds__(kThreadsTc, 1) moe_prefill_tc_kernel(TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint64_t* full = bars;                        // [kSStages] producer -> transform/MMA
    uint64_t* sempty = full + kSStages;           // [kSStages] MMA -> producer
    uint64_t* aready = sempty + kSStages;         // [kAStages] transform -> MMA
    uint64_t* aempty = aready + kAStages;         // [kAStages] MMA -> transform
    uint64_t* accfull = aempty + kAStages;        // MMA -> epilogue
    uint64_t* accempty = accfull + 1;             // epilogue -> MMA
    uint64_t* drained = accempty + 1;             // MMA: all issued MMAs complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&full[s], kProducerThreads + 1);
            mbar_init(&sempty[s], 1);
        }
        for (int s = 0; s < kAStages; ++s) {
            mbar_init(&aready[s], kTransformWarps);
            mbar_init(&aempty[s], 1);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, kTransformWarps);
        mbar_init(drained, 1);
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
        const int q = warp & 3, rt2 = warp >> 2;
        const int m = 32 * q + lane;                 // row within the 128-row tile
        const int sub = m >> 4, gi = m & 7, isb = (m >> 3) & 1;
        const uint32_t mask = isb ? 0x00F000F0u : 0x000F000Fu;
        const uint32_t mul = isb ? 0x2C002C00u : 0x3C003C00u;   // 1/16 : 1
        const uint32_t add = isb ? 0xD480D480u : 0xE408E408u;   // -72 : -1032
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        uint32_t it = 0, icount = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int4 tile = a.tiles[item / a.RT2];
            const int pair = item % a.RT2;
            const int n = tile.z, start = tile.y, nm = (n + 15) & ~15;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kSStages, sa = it % kAStages;
                if (!tc_wait_warp(&full[s], (it / kSStages) & 1, abort_flag, a.err, 21)) { ok = false; break; }
                if (!tc_wait_warp(&aempty[sa], ((it / kAStages) & 1) ^ 1, abort_flag, a.err, 22)) { ok = false; break; }
                tc_fence_after();
                const uint8_t* blk = sm + kOffW + s * kWStageBytes + rt2 * kBlockBytes;
                const uint8_t* rowp = blk + sub * 512 + gi * 64;  // lanes 4gi..4gi+3 of the sub-tile
                uint4 wv[4];
#pragma unroll
                for (int ti = 0; ti < 4; ++ti) wv[ti] = *reinterpret_cast<const uint4*>(rowp + 16 * ti);
                const uint32_t sp = *reinterpret_cast<const uint32_t*>(blk + kNibbleBytes + sub * 32 + gi * 4);
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
                const uint32_t ta = tmem + lane_base + kABase + 64 * sa + 32 * rt2;
                tc_st16(ta, r);
                tc_st16(ta + 16, r + 16);
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[sa]);
            }
            if (!ok) break;
            // ---------------------------------------------------- epilogue
            if (!tc_wait_warp(accfull, icount & 1, abort_flag, a.err, 23)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tacc = tmem + lane_base + kAccBase + rt2 * kAccCols;
            const int row = (2 * pair + rt2) * 128 + m;  // row of the weight matrix
            for (int c16 = 0; c16 < nm; c16 += 16) {
                uint32_t v[16];
                tc_ld16_wait(tacc + c16, v);
                if (kPhase == 0) {
                    // gate row (isb = 0) and up row (isb = 1) of the same h index sit 8 lanes apart:
                    // the gate lane forms h for even tokens, the up lane for odd ones.
                    const int j = (row >> 4) * 8 + (row & 7);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float send = __uint_as_float(isb ? v[2 * i] : v[2 * i + 1]);
                        const float recv = __shfl_xor_sync(0xffffffffu, send, 8);
                        const float g = isb ? recv : __uint_as_float(v[2 * i]);
                        const float u = isb ? __uint_as_float(v[2 * i + 1]) : recv;
                        const int nn = c16 + 2 * i + isb;
                        if (nn < n) {
                            const float4 si = a.slot[start + nn];
                            const float hv = silu_f(g * si.x) * (u * si.x);
                            a.h16[(size_t)(start + nn) * a.I + j] = __float2half_rn(hv * si.y);
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int nn = c16 + i;
                        if (nn < n) {
                            const float4 si = a.slot[start + nn];
                            const int t = __float_as_int(si.w);
                            atomicAdd(a.y32 + (size_t)t * a.H + row, __uint_as_float(v[i]) * si.z);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty);
            ++icount;
        }
    } else if (warp < kMmaWarp) {
        // ------------------------------------------------------- producer
        // Thread tid copies 16-byte chunk (tid & 7) of rows tid/8, tid/8 + 8, ...
        constexpr int kRowsPer = kTcMaxTok / (kProducerThreads / 8);  // 16
        const int tid = threadIdx.x - kTransformWarps * 32;
        const int chunk = tid & 7, r0 = tid >> 3;
        uint32_t it = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int4 tile = a.tiles[item / a.RT2];
            const int pair = item % a.RT2;
            const int n = tile.z, start = tile.y;
            int64_t off[kRowsPer];
#pragma unroll
            for (int i = 0; i < kRowsPer; ++i) {
                const int r = r0 + 8 * i;
                off[i] = r < n ? (kPhase == 0 ? (int64_t)a.tok[start + r] : (int64_t)(start + r)) * a.src_pitch : 0;
            }
            const uint8_t* w0 = a.weights + (size_t)tile.x * a.expert_stride + a.mat_offset +
                                (size_t)(2 * pair) * KB * kBlockBytes;
            const uint8_t* w1 = w0 + (size_t)KB * kBlockBytes;
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kSStages;
                if (!tc_wait(&sempty[s], ((it / kSStages) & 1) ^ 1, abort_flag, a.err, 24)) { ok = false; break; }
                uint8_t* wdst = sm + kOffW + s * kWStageBytes;
                if (tid == 0) {
                    mbar_arrive_expect_tx(&full[s], 2 * kBlockBytes);
                    bulk_g2s(wdst, w0 + (size_t)kb * kBlockBytes, kBlockBytes, &full[s]);
                    bulk_g2s(wdst + kBlockBytes, w1 + (size_t)kb * kBlockBytes, kBlockBytes, &full[s]);
                }
                const uint32_t bdst = smem_addr(sm + kOffB + s * kBTileBytes) + ((r0 & 7) << 7) + ((chunk ^ (r0 & 7)) << 4);
                const __half* src = a.src + (size_t)kb * 64 + chunk * 8;
#pragma unroll
                for (int i = 0; i < kRowsPer; ++i) {
                    const int r = r0 + 8 * i;  // r & 7 == r0 & 7: same swizzle for every row of this thread
                    if (r < n) cp_async16(bdst + (r >> 3) * 1024, src + off[i]);
                }
                cp_async_mbar_arrive(&full[s]);
            }
        }
        cp_async_wait_all();
        if (tid == 0) {
            // bulk copies still in flight (after an abort) must land before the CTA exits
            const uint32_t first = it > (uint32_t)kSStages ? it - kSStages : 0;
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t k = first; k < it; ++k) {
                while (!mbar_try_wait(&full[k % kSStages], (k / kSStages) & 1) && globaltimer_ns() - t0 < kTcWaitNs) {
                }
            }
        }
        __syncwarp();
    } else {
      if (lane == 0) {
        // ------------------------------------------------------------ MMA
        uint32_t it = 0, icount = 0;
        bool ok = true, issued = false;
        for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
            const int4 tile = a.tiles[item / a.RT2];
            const int nm = (tile.z + 15) & ~15;
            const uint32_t idesc = tc_idesc_f16(nm, false);
            if (!tc_wait(accempty, (icount & 1) ^ 1, abort_flag, a.err, 25)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < KB; ++kb, ++it) {
                const int s = it % kSStages, sa = it % kAStages;
                if (!tc_wait(&full[s], (it / kSStages) & 1, abort_flag, a.err, 26)) { ok = false; break; }
                if (!tc_wait(&aready[sa], (it / kAStages) & 1, abort_flag, a.err, 27)) { ok = false; break; }
                fence_proxy_async_smem();
                tc_fence_after();
                const uint64_t bdesc = tc_sdesc_sw128(smem_addr(sm + kOffB + s * kBTileBytes));
#pragma unroll
                for (int t2 = 0; t2 < 2; ++t2) {
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        tc_mma_ts(tmem + kAccBase + t2 * kAccCols, tmem + kABase + 64 * sa + 32 * t2 + 8 * j, bdesc + 2 * j, idesc,
                                  (kb | j) != 0);
                }
                issued = true;
                tc_commit(&sempty[s]);
                tc_commit(&aempty[sa]);
            }
            if (!ok) break;
            tc_commit(accfull);
            ++icount;
        }
        if (issued) {
            // every MMA must complete before the tensor memory is released
            tc_commit(drained);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(drained, 0) && globaltimer_ns() - t0 < kTcWaitNs) {
            }
        }
      }
      __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tc_dealloc(tmem, kTmemCols);
}

// One warp per token: max |x_t|, the power-of-two scales, x16 = fp16(x * 2^e).
__global__ void prefill_prep_kernel(const __nv_bfloat16* __restrict__ x, int T, int H, const float* __restrict__ meta,
                                    __half* __restrict__ x16, float4* __restrict__ tscale) {
    const int lane = threadIdx.x & 31;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const double bound = (double)meta[0] * (1.0 + 1e-3);  // max_j L1(gate_j) L1(up_j), with rounding margin
    for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
        const uint4* row = reinterpret_cast<const uint4*>(x + (size_t)t * H);
        float mx = 0.0f;
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = row[i];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                mx = fmaxf(mx, fabsf(__uint_as_float(w[k] << 16)));
                mx = fmaxf(mx, fabsf(__uint_as_float(w[k] & 0xFFFF0000u)));
            }
        }
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        int e = 0, f = 0;
        if (mx > 0.0f && mx <= 3.0e38f) {
            e = min(120, max(-120, 14 - ilogbf(mx)));
            const double hb = bound * (double)mx * (double)mx;
            if (hb > 0.0) f = min(120, max(-120, ilogb(16384.0 / hb)));
        }
        uint4* out = reinterpret_cast<uint4*>(x16 + (size_t)t * H);
        for (int i = lane; i < H / 8; i += 32) {
            const uint4 v = row[i];
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o4[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const __half lo = __float2half_rn(ldexpf(__uint_as_float(w[k] << 16), e));
                const __half hi = __float2half_rn(ldexpf(__uint_as_float(w[k] & 0xFFFF0000u), e));
                o4[k] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
            }
            out[i] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
        }
        if (lane == 0) tscale[t] = make_float4(ldexpf(1.0f, -e), ldexpf(1.0f, f), ldexpf(1.0f, -f), 0.0f);
    }
}

// Per-position epilogue factors and the tile list (one CTA). Tiles hold at
// most kTcMaxTok tokens of one expert and are ordered by decreasing size.
__global__ void __launch_bounds__(1024) prefill_plan_kernel(Plan p, int T, int K, int S, const float4* __restrict__ tscale,
                                                            float4* __restrict__ slot, int4* __restrict__ tiles,
                                                            int* __restrict__ n_tiles) {
    __shared__ int bcnt[kTcMaxTok / 16], bbase[kTcMaxTok / 16], bcur[kTcMaxTok / 16];
    constexpr int NB = kTcMaxTok / 16;
    const int TK = T * K;
    for (int i = threadIdx.x; i < TK; i += blockDim.x) {
        const int t = i / K;
        const float4 ts = tscale[t];
        slot[p.pos[i]] = make_float4(ts.x, ts.y, p.w[i] * ts.z, __int_as_float(t));
    }
    for (int i = threadIdx.x; i < S * T; i += blockDim.x) {
        const int t = i % T;
        const float4 ts = tscale[t];
        slot[TK + i] = make_float4(ts.x, ts.y, ts.z, __int_as_float(t));
    }
    if (threadIdx.x < NB) bcnt[threadIdx.x] = bcur[threadIdx.x] = 0;
    __syncthreads();
    const int na = *p.n_active;
    for (int pass = 0; pass < 2; ++pass) {
        for (int u = threadIdx.x; u < na; u += blockDim.x) {
            const int cnt = p.act_cnt[u];
            if (cnt <= 0) continue;
            const int nt = (cnt + kTcMaxTok - 1) / kTcMaxTok;
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

__global__ void prefill_out_kernel(const float* __restrict__ y32, const float* __restrict__ residual, size_t n,
                                   __nv_bfloat16* __restrict__ y) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x) {
        float4 v = reinterpret_cast<const float4*>(y32)[i];
        if (residual) {
            const float4 r = reinterpret_cast<const float4*>(residual)[i];
            v.x += r.x; v.y += r.y; v.z += r.z; v.w += r.w;
        }
        __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 o;
        o.x = *reinterpret_cast<uint32_t*>(&lo);
        o.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(y)[i] = o;
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

cudaError_t launch_prefill_prep(const void* x, int T, int H, const float* meta, __half* x16, float4* tscale,
                                cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int grid = (T + 7) / 8 < 1184 ? (T + 7) / 8 : 1184;
    prefill_prep_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, T, H, meta, x16, tscale);
    return cudaGetLastError();
}

cudaError_t launch_prefill_plan(const Plan& p, int T, int K, int S, const float4* tscale, float4* slot, int4* tiles,
                                int* n_tiles, cudaStream_t st) {
    prefill_plan_kernel<<<1, 1024, 0, st>>>(p, T, K, S, tscale, slot, tiles, n_tiles);
    return cudaGetLastError();
}

cudaError_t launch_prefill_gemm(int phase, const uint8_t* weights, const Dims& d, const __half* src, const Plan& p,
                                const float4* slot, const int4* tiles, const int* n_tiles, __half* h16, float* y32,
                                int* err, int n_sm, cudaStream_t st) {
    TcArgs a;
    a.weights = weights;
    a.expert_stride = d.expert_stride;
    a.mat_offset = phase == 0 ? 0 : d.gu_bytes;
    a.KB = phase == 0 ? d.H / kGroup : d.I / kGroup;
    a.RT2 = phase == 0 ? (2 * d.I / kTileRows) / 2 : (d.H / kTileRows) / 2;
    a.src = src;
    a.src_pitch = phase == 0 ? d.H : d.I;
    a.tok = p.tok;
    a.slot = slot;
    a.tiles = tiles;
    a.n_tiles = n_tiles;
    a.h16 = h16;
    a.y32 = y32;
    a.I = d.I;
    a.H = d.H;
    a.err = err;
    cudaError_t e;
    if (phase == 0) {
        e = cudaFuncSetAttribute(moe_prefill_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
        if (e != cudaSuccess) return e;
        moe_prefill_tc_kernel<0><<<n_sm, kThreadsTc, kSmemTc, st>>>(a);
    } else {
        e = cudaFuncSetAttribute(moe_prefill_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTc);
        if (e != cudaSuccess) return e;
        moe_prefill_tc_kernel<1><<<n_sm, kThreadsTc, kSmemTc, st>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_prefill_out(const float* y32, const float* residual, int T, int H, void* y, cudaStream_t st) {
    const size_t n = (size_t)T * H;
    if (n == 0) return cudaSuccess;
    const size_t blocks = (n / 4 + 255) / 256;
    prefill_out_kernel<<<(int)(blocks < 4736 ? blocks : 4736), 256, 0, st>>>(y32, residual, n, (__nv_bfloat16*)y);
    return cudaGetLastError();
}

}  // namespace coli
