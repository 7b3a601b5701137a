// ffn_core.cu -- int4 expert matrices on the CUDA cores (fp32 arithmetic).
//
// The routed experts' three matrices (gate, up, down) are streamed from HBM
// once per forward for every active expert of the batch-union ("Colibri: 2400
// lines of pure C ...", kechuai.cn, section 二: each unique expert is read
// once per batch; the batch-1 matvec in fp32 beat the int4 SIMD kernel on the
// CPU, colibri daily, jsqmd.com, section 四 highlight 4).
//
// Work item = (chunk of up to kTB tokens of an active expert, 128-row tile),
// so an expert with many tokens (the shared one) spreads over many CTAs. A
// CTA of 8 warps owns one tile;
// warp w owns 16-row sub-tile w and streams its 512 + 32 bytes per 64-input
// group with 128-bit non-allocating loads, NP groups in flight. Each lane
// turns a nibble into an exact float with one LOP3 (the nibble is OR-ed into
// the mantissa of 2^23) and one packed FFMA2 that removes the 2^23 bias, the
// nibble's bit position and the +8 offset at once; the dot products run on
// packed FFMA2 with per-group accumulators scaled by the group's fp16 scale.
#include "common.cuh"
#include "kernels.cuh"
#include "int4_math.cuh"

namespace coli {

constexpr int kThreads = 256;  // 8 warps = 8 sub-tiles of one 128-row tile
constexpr int kTB = kCoreTok;  // tokens per pass over the weights (one work item)
constexpr int kNP = 8;         // groups in flight per warp

// Issue the loads of the first kNP groups of this warp's sub-tile of a
// 128-row tile (called before the item's inputs are staged, so their latency
// overlaps the staging).
__device__ __forceinline__ void tile_prefetch(const uint8_t* __restrict__ tile, int G, uint4 wb[kNP], uint32_t sb[kNP]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2;
    const uint8_t* wp = tile + warp * 512 + lane_slot(lane) * 16;
    const uint8_t* sp = tile + kNibbleBytes + warp * 32 + gi * 4;
#pragma unroll
    for (int i = 0; i < kNP; ++i) {
        if (i < G) {
            wb[i] = ldg_stream(wp + (size_t)i * kBlockBytes);
            sb[i] = ldg_stream32(sp + (size_t)i * kBlockBytes);
        }
    }
}

// One 128-row tile of an int4 matrix times up to kTB staged input rows, the
// first kNP groups already loaded by tile_prefetch. Returns, per token, the
// fp32 results of rows gi (acc0) and gi+8 (acc1) of this warp's sub-tile,
// summed over the four lanes of the row (valid in all).
__device__ __forceinline__ void tile_dot(const uint8_t* __restrict__ tile, int G, const float4* xs, int nt,
                                         float acc0[kTB], float acc1[kTB], uint4 wb[kNP], uint32_t sb[kNP]) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2, ti = lane & 3;
    const uint8_t* wp = tile + warp * 512 + lane_slot(lane) * 16;
    const uint8_t* sp = tile + kNibbleBytes + warp * 32 + gi * 4;
#pragma unroll
    for (int tb = 0; tb < kTB; ++tb) { acc0[tb] = 0.0f; acc1[tb] = 0.0f; }
    for (int g0 = 0; g0 < G; g0 += kNP) {
#pragma unroll
        for (int i = 0; i < kNP; ++i) {
            const int g = g0 + i;
            if (g < G) {
                const uint4 wv = wb[i];
                const uint32_t sv = sb[i];
                if (g + kNP < G) {
                    wb[i] = ldg_stream(wp + (size_t)(g + kNP) * kBlockBytes);
                    sb[i] = ldg_stream32(sp + (size_t)(g + kNP) * kBlockBytes);
                }
                group_dot<kTB>(wv, sv, xs + g * 16, G * 16, ti, nt, acc0, acc1);
            }
        }
    }
#pragma unroll
    for (int tb = 0; tb < kTB; ++tb) {
        acc0[tb] += __shfl_xor_sync(0xffffffffu, acc0[tb], 1);
        acc0[tb] += __shfl_xor_sync(0xffffffffu, acc0[tb], 2);
        acc1[tb] += __shfl_xor_sync(0xffffffffu, acc1[tb], 1);
        acc1[tb] += __shfl_xor_sync(0xffffffffu, acc1[tb], 2);
    }
}

// Active expert owning global chunk c: the last a with act_chunk[a] <= c.
__device__ __forceinline__ int chunk_owner(const int32_t* __restrict__ act_chunk, int n_active, int c) {
    int lo = 0, hi = n_active - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(act_chunk + mid) <= c) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Gate/up + SwiGLU. Item = (chunk of an active expert a, 128-row tile rt of the [2I][H]
// interleaved gate/up matrix). h[pos][j] = silu(g_j) * u_j.
template <typename XT>
__global__ void __launch_bounds__(kThreads, 2) gateup_core_kernel(const uint8_t* __restrict__ weights, Dims d,
                                                               const XT* __restrict__ x, Plan p, float* __restrict__ h) {
    extern __shared__ float4 xs[];
    __shared__ int32_t rows[kTB];
    const int G = d.H / kGroup;
    const int RT = 2 * d.I / kTileRows;
    const int n_active = *p.n_active;
    const int n_items = p.act_chunk[n_active] * RT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2, ti = lane & 3;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int c = item / RT, rt = item - c * RT;
        const int a = chunk_owner(p.act_chunk, n_active, c);
        const int ex = p.act_expert[a], off = p.act_off[a], cnt = p.act_cnt[a];
        const uint8_t* tile = weights + expert_offset(d, ex) + (size_t)rt * G * kBlockBytes;
        const int j = (rt * 8 + warp) * 8 + gi;  // gate row of this lane's row gi
        const int t0 = (c - p.act_chunk[a]) * kTB;
        {
            const int nt = min(kTB, cnt - t0);
            uint4 wb[kNP];
            uint32_t sb[kNP];
            tile_prefetch(tile, G, wb, sb);
            __syncthreads();
            if (threadIdx.x < nt) rows[threadIdx.x] = p.tok[off + t0 + threadIdx.x];
            __syncthreads();
            stage_rows<XT>(xs, x, rows, nt, d.H, threadIdx.x, blockDim.x);
            __syncthreads();
            float g_acc[kTB], u_acc[kTB];
            tile_dot(tile, G, xs, nt, g_acc, u_acc, wb, sb);
            if (ti == 0) {
#pragma unroll
                for (int tb = 0; tb < kTB; ++tb)
                    if (tb < nt) h[(size_t)(off + t0 + tb) * d.I + j] = silu_f(g_acc[tb]) * u_acc[tb];
            }
        }
    }
}

// Down. Item = (active expert a, 128-row tile rt of [H][I]). o[pos][r].
__global__ void __launch_bounds__(kThreads, 2) down_core_kernel(const uint8_t* __restrict__ weights, Dims d,
                                                             const float* __restrict__ h, Plan p, float* __restrict__ o) {
    extern __shared__ float4 xs[];
    __shared__ int32_t rows[kTB];
    const int G = d.I / kGroup;
    const int RT = d.H / kTileRows;
    const int n_active = *p.n_active;
    const int n_items = p.act_chunk[n_active] * RT;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gi = lane >> 2, ti = lane & 3;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int c = item / RT, rt = item - c * RT;
        const int a = chunk_owner(p.act_chunk, n_active, c);
        const int ex = p.act_expert[a], off = p.act_off[a], cnt = p.act_cnt[a];
        const uint8_t* tile = weights + expert_offset(d, ex) + d.gu_bytes + (size_t)rt * G * kBlockBytes;
        const int r0 = rt * kTileRows + warp * kSubRows + gi;
        const int t0 = (c - p.act_chunk[a]) * kTB;
        {
            const int nt = min(kTB, cnt - t0);
            uint4 wb[kNP];
            uint32_t sb[kNP];
            tile_prefetch(tile, G, wb, sb);
            __syncthreads();
            if (threadIdx.x < nt) rows[threadIdx.x] = off + t0 + threadIdx.x;  // h is indexed by position
            __syncthreads();
            stage_rows<float>(xs, h, rows, nt, d.I, threadIdx.x, blockDim.x);
            __syncthreads();
            float a0[kTB], a1[kTB];
            tile_dot(tile, G, xs, nt, a0, a1, wb, sb);
            if (ti == 0) {
#pragma unroll
                for (int tb = 0; tb < kTB; ++tb) {
                    if (tb < nt) {
                        o[(size_t)(off + t0 + tb) * d.H + r0] = a0[tb];
                        o[(size_t)(off + t0 + tb) * d.H + r0 + 8] = a1[tb];
                    }
                }
            }
        }
    }
}

static int grid_items(int max_items, int n_sm, int per_sm) {
    int g = n_sm * per_sm;
    return max_items < g ? (max_items < 1 ? 1 : max_items) : g;
}

cudaError_t launch_gateup_core(const uint8_t* weights, const Dims& d, const void* x, coli_dtype dt, int T,
                               const Plan& p, float* h, int max_active, int n_sm, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const size_t smem = (size_t)kTB * d.H * sizeof(float);
    const int grid = grid_items(max_active * (2 * d.I / kTileRows), n_sm, 2);
    cudaError_t e;
    if (dt == COLI_F32) {
        e = cudaFuncSetAttribute(gateup_core_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        gateup_core_kernel<float><<<grid, kThreads, smem, st>>>(weights, d, (const float*)x, p, h);
    } else {
        e = cudaFuncSetAttribute(gateup_core_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        gateup_core_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(weights, d, (const __nv_bfloat16*)x, p, h);
    }
    return cudaGetLastError();
}

cudaError_t launch_down_core(const uint8_t* weights, const Dims& d, const float* h, int T, const Plan& p, float* o,
                             int max_active, int n_sm, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const size_t smem = (size_t)kTB * d.I * sizeof(float);
    const int grid = grid_items(max_active * (d.H / kTileRows), n_sm, 2);
    cudaError_t e = cudaFuncSetAttribute(down_core_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    down_core_kernel<<<grid, kThreads, smem, st>>>(weights, d, h, p, o);
    return cudaGetLastError();
}

}  // namespace coli
