// router.cu -- router GEMV (fp64 accumulation), top-k selection with
// softmax renormalisation, and the batch-union planner.
//
// Router: "Colibri: 2400 lines of pure C ..." (kechuai.cn), section 一: each
// layer routes a token to 8 of its 256 experts. Batch-union: same page,
// section 二: the positions of a batch read each unique expert once.
#include "common.cuh"
#include "kernels.cuh"
#include "topk.cuh"

namespace coli {

// ---------------------------------------------------------------------------
// Router logits: l[t][e] = sum_h Wr[e][h] x[t][h] + b[e], accumulated in fp64.
// Products of two fp32 (or bf16 x fp32) values are exact in fp64, so the
// logits agree with an fp64 reference up to summation order (~1e-16
// relative): the top-k ids are then reproducible bit for bit.
//
// Grid (ceil(E/2), ceil(T/kRouterTok)); 256 threads: warp w handles expert
// 2*blockIdx.x + w/4 and quarter (w%4) of H for up to kRouterTok tokens; the
// four quarters are summed in a fixed order through shared memory.
// ---------------------------------------------------------------------------
constexpr int kRouterTok = 4;

template <typename XT>
__device__ __forceinline__ void load4(const XT* p, double v[4]);

template <>
__device__ __forceinline__ void load4<float>(const float* p, double v[4]) {
    float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, double v[4]) {
    uint2 u = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
}

template <typename XT>
__global__ void __launch_bounds__(256) router_logits_kernel(const float* __restrict__ wr, const float* __restrict__ bias,
                                                            const XT* __restrict__ x, int T, int H, int E,
                                                            double* __restrict__ logits) {
    __shared__ double part[8][kRouterTok];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 2 + (warp >> 2);
    const int quarter = warp & 3;
    const int t0 = blockIdx.y * kRouterTok;
    const int nt = min(kRouterTok, T - t0);
    const int seg = H / 4;
    double acc[kRouterTok];
#pragma unroll
    for (int j = 0; j < kRouterTok; ++j) acc[j] = 0.0;
    if (e < E) {
        const float* wrow = wr + (size_t)e * H + quarter * seg;
        for (int i = lane * 4; i < seg; i += 128) {
            float4 w4 = *reinterpret_cast<const float4*>(wrow + i);
            double wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int j = 0; j < kRouterTok; ++j) {
                if (j < nt) {
                    double xv[4];
                    load4<XT>(x + (size_t)(t0 + j) * H + quarter * seg + i, xv);
                    acc[j] = fma(wd[0], xv[0], acc[j]);
                    acc[j] = fma(wd[1], xv[1], acc[j]);
                    acc[j] = fma(wd[2], xv[2], acc[j]);
                    acc[j] = fma(wd[3], xv[3], acc[j]);
                }
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kRouterTok; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
        for (int j = 0; j < kRouterTok; ++j) part[warp][j] = acc[j];
    }
    __syncthreads();
    if (threadIdx.x < 2 * kRouterTok) {
        int ew = threadIdx.x / kRouterTok, j = threadIdx.x % kRouterTok;
        int ee = blockIdx.x * 2 + ew;
        if (ee < E && j < nt) {
            double s = ((part[ew * 4 + 0][j] + part[ew * 4 + 1][j]) + part[ew * 4 + 2][j]) + part[ew * 4 + 3][j];
            logits[(size_t)(t0 + j) * E + ee] = s + (bias ? (double)bias[ee] : 0.0);
        }
    }
}

// ---------------------------------------------------------------------------
// Router logits for token batches: the same fp64 sums as a blocked GEMM.
// CTA tile 64 tokens x 128 experts, 128 threads; thread (ty, tx) owns tokens
// 8ty..8ty+7 and experts tx + 16j (j < 8): 64 fp64 accumulators. 16-input
// chunks of x and Wr are widened to fp64 in shared memory (double-buffered;
// the next chunk is fetched into registers while the current one is
// multiplied). The input dimension may be split into `nsplit` ranges
// (blockIdx.z) whose partial sums land in part[z] and are added in a fixed
// order by router_reduce_kernel, so the result does not depend on timing.
// ---------------------------------------------------------------------------
constexpr int kRgT = 64, kRgE = 128, kRgK = 16;

template <typename XT>
__device__ __forceinline__ void rg_load8(const XT* p, float v[8]);
template <>
__device__ __forceinline__ void rg_load8<float>(const float* p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void rg_load8<__nv_bfloat16>(const __nv_bfloat16* p, float v[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <typename XT>
__global__ void __launch_bounds__(128) router_gemm_kernel(const float* __restrict__ wr, const float* __restrict__ bias,
                                                          const XT* __restrict__ x, int T, int H, int E, int nsplit,
                                                          double* __restrict__ out) {
    __shared__ __align__(16) double xs[2][kRgK][kRgT];   // 16 KB
    __shared__ __align__(16) double ws[2][kRgK][kRgE];   // 32 KB
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.x * kRgT, e0 = blockIdx.y * kRgE;
    const int hspan = H / nsplit, h0 = blockIdx.z * hspan;
    // loaders: x row tid/2, inputs 8 (tid & 1) .. +7; Wr row tid, inputs 0..15
    const int xr = tid >> 1, xk = (tid & 1) * 8;
    const bool xok = t0 + xr < T, wok = e0 + tid < E;
    const XT* xp = x + (size_t)(xok ? t0 + xr : 0) * H + h0 + xk;
    const float* wp = wr + (size_t)(wok ? e0 + tid : 0) * H + h0;
    float xv[8], wv[16];
    auto fetch = [&](int k0) {
        if (xok) {
            rg_load8<XT>(xp + k0, xv);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) xv[i] = 0.0f;
        }
        if (wok) {
            rg_load8<float>(wp + k0, wv);
            rg_load8<float>(wp + k0 + 8, wv + 8);
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) wv[i] = 0.0f;
        }
    };
    auto stash = [&](int b) {
#pragma unroll
        for (int i = 0; i < 8; ++i) xs[b][xk + i][xr] = (double)xv[i];
#pragma unroll
        for (int i = 0; i < 16; ++i) ws[b][i][tid] = (double)wv[i];
    };
    double acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
    fetch(0);
    stash(0);
    __syncthreads();
    const int nk = hspan / kRgK;
    for (int c = 0; c < nk; ++c) {
        const int b = c & 1;
        if (c + 1 < nk) fetch((c + 1) * kRgK);
#pragma unroll 4
        for (int k = 0; k < kRgK; ++k) {
            double xr8[8], wc[8];
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const double2 v = *reinterpret_cast<const double2*>(&xs[b][k][ty * 8 + i]);
                xr8[i] = v.x;
                xr8[i + 1] = v.y;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) wc[j] = ws[b][k][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] = fma(xr8[i], wc[j], acc[i][j]);
        }
        if (c + 1 < nk) stash(b ^ 1);
        __syncthreads();
    }
    double* dst = out + (size_t)blockIdx.z * T * E;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + ty * 8 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int e = e0 + tx + 16 * j;
            if (e < E) dst[(size_t)t * E + e] = acc[i][j] + ((nsplit == 1 && bias) ? (double)bias[e] : 0.0);
        }
    }
}

// logits = sum over splits s = 0, 1, ... of part[s] (in that order) + bias.
__global__ void router_reduce_kernel(const double* __restrict__ part, const float* __restrict__ bias, int T, int E,
                                     int nsplit, double* __restrict__ logits) {
    const size_t n = (size_t)T * E;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        double v = part[i];
        for (int s = 1; s < nsplit; ++s) v += part[(size_t)s * n + i];
        logits[i] = v + (bias ? (double)bias[i % E] : 0.0);
    }
}

// ---------------------------------------------------------------------------
// Top-k. Lane l of a warp holds the logits of experts l, l+32, ...; K rounds
// each take the best remaining (largest logit, ties to the lower id); weights
// are the softmax over the K selected logits, in fp64, fixed summation order.
// ---------------------------------------------------------------------------
// ---------------------------------------------------------------------------
// Top-k: one warp per token (warp_topk in topk.cuh).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) topk_kernel(const double* __restrict__ logits, int T, int E, int K,
                                                   double topp, int e_lo, int e_hi, int32_t* __restrict__ ids,
                                                   float* __restrict__ w) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    int id;
    float wt;
    if (E <= 256) warp_topk8<false>(logits + (size_t)t * E, E, K, topp, lane, &id, &wt);
    else warp_topk<false>(logits + (size_t)t * E, E, K, topp, lane, &id, &wt);
    if (lane < K) {
        // experts outside [e_lo, e_hi) belong to another rank: an empty slot here
        ids[(size_t)t * K + lane] = (id >= e_lo && id < e_hi) ? id : -1;
        w[(size_t)t * K + lane] = wt;
    }
}

// ---------------------------------------------------------------------------
// Batch-union planner, one CTA of 1024 threads. For the T*K routed slots:
//   cnt[e], off = exclusive scan, unique = {e : cnt[e] > 0} ascending,
//   pos[t][k] = off[e] + (rank of t among e's tokens, ascending t),
//   tok[pos] = t,
// then the active-expert list (unique experts, then the S shared experts,
// each shared expert taking all T tokens at positions T*K + j*T + t).
// Deterministic: positions come from per-warp counts over token chunks and a
// sequential walk inside each chunk, never from atomics.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;

__global__ void __launch_bounds__(kPlanThreads) plan_kernel(const int32_t* __restrict__ ids, int T, int K, int E, int S,
                                                            Plan p) {
    extern __shared__ int32_t sm[];
    int32_t* wcnt = sm;                          // [kPlanWarps][E]  -> per-warp cursor
    int32_t* off = wcnt + kPlanWarps * E;        // [E+1]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = (T + kPlanWarps - 1) / kPlanWarps;
    const int tb = warp * chunk, te = min(T, tb + chunk);

    // A warp walks its chunk 32 / K tokens at a time: lane l holds slot l % K of
    // token l / K, so lane order is (token, slot) order, and one coalesced load
    // (issued an iteration ahead) brings the ids of every token of the step.
    const int tpi = 32 / K, li = lane / K, lk = lane % K;
    auto slot_id = [&](int t0) { return (li < tpi && t0 + li < te) ? __ldg(ids + (size_t)(t0 + li) * K + lk) : -2; };
    for (int i = threadIdx.x; i < kPlanWarps * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    // per-warp counts over its token chunk; lanes holding the same expert add as one (e < 0: an
    // empty slot, or no slot)
    {
        int e_next = slot_id(tb);
        for (int t0 = tb; t0 < te; t0 += tpi) {
            const int e = e_next;
            e_next = slot_id(t0 + tpi);
            const unsigned m = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(m) - 1) wcnt[warp * E + e] += __popc(m);
        }
    }
    __syncthreads();
    // per expert: exclusive scan over warps -> warp cursor base, total count
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
        for (int w = 0; w < kPlanWarps; ++w) {
            int c = wcnt[w * E + e];
            wcnt[w * E + e] = run;
            run += c;
        }
        off[e + 1] = run;  // count for now
    }
    __syncthreads();
    // exclusive scan of counts over experts (E <= 1024: one thread each, Hillis-Steele)
    if (threadIdx.x == 0) off[0] = 0;
    int cnt_e = 0;
    if (threadIdx.x < E) cnt_e = off[threadIdx.x + 1];
    __syncthreads();
    // inclusive scan in place over off[1..E]
    for (int d = 1; d < E; d <<= 1) {
        int add = 0;
        if (threadIdx.x < E && threadIdx.x >= d) add = off[threadIdx.x + 1 - d];
        __syncthreads();
        if (threadIdx.x < E) off[threadIdx.x + 1] += add;
        __syncthreads();
    }
    if (threadIdx.x < E) {
        p.cnt[threadIdx.x] = cnt_e;
        p.off[threadIdx.x] = off[threadIdx.x];
    }
    if (threadIdx.x == 0) p.off[E] = off[E];
    // unique list: rank among experts with cnt > 0
    __shared__ int32_t flag_scan[1024];
    if (threadIdx.x < 1024) flag_scan[threadIdx.x] = (threadIdx.x < E && cnt_e > 0) ? 1 : 0;
    __syncthreads();
    for (int d = 1; d < 1024; d <<= 1) {
        int add = (threadIdx.x >= d) ? flag_scan[threadIdx.x - d] : 0;
        __syncthreads();
        flag_scan[threadIdx.x] += add;
        __syncthreads();
    }
    const int n_unique = flag_scan[1023];
    if (threadIdx.x < E && cnt_e > 0) {
        int r = flag_scan[threadIdx.x] - 1;
        p.unique[r] = threadIdx.x;
        p.act_expert[r] = threadIdx.x;
        p.act_off[r] = off[threadIdx.x];
        p.act_cnt[r] = cnt_e;
    }
    if (threadIdx.x < S) {
        int r = n_unique + threadIdx.x;
        p.act_expert[r] = E + threadIdx.x;
        p.act_off[r] = T * K + threadIdx.x * T;
        p.act_cnt[r] = T;
    }
    if (threadIdx.x == 0) {
        *p.n_unique = n_unique;
        *p.n_active = n_unique + S;
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // chunks of kCoreTok tokens per active expert, prefix (work items of the CUDA-core kernels)
        int run = 0;
        for (int a = 0; a < n_unique + S; ++a) {
            p.act_chunk[a] = run;
            run += (p.act_cnt[a] + kCoreTok - 1) / kCoreTok;
        }
        p.act_chunk[n_unique + S] = run;
    }
    // positions: each warp walks its chunk in (token, slot) order; lanes holding the same
    // expert take consecutive positions in lane order, then the lowest of them advances the cursor
    {
        int e_next = slot_id(tb);
        for (int t0 = tb; t0 < te; t0 += tpi) {
            const int e = e_next;
            e_next = slot_id(t0 + tpi);
            const int t = t0 + li;
            const unsigned m = __match_any_sync(0xffffffffu, e);
            if (e >= 0) {
                const int q = off[e] + wcnt[warp * E + e] + __popc(m & ((1u << lane) - 1u));
                p.pos[(size_t)t * K + lk] = q;
                p.tok[q] = t;
            } else if (e == -1) {
                p.pos[(size_t)t * K + lk] = -1;  // an empty slot
            }
            __syncwarp();
            if (e >= 0 && lane == __ffs(m) - 1) wcnt[warp * E + e] += __popc(m);
            __syncwarp();
        }
    }
    // shared experts: all tokens in order
    for (int i = threadIdx.x; i < S * T; i += blockDim.x) p.tok[T * K + i] = i % T;
}

// ---------------------------------------------------------------------------
// Host launchers.
// ---------------------------------------------------------------------------
// Split of the input dimension for the blocked router GEMM (0: the GEMV
// kernel serves this call): split until about two CTAs per SM are busy.
static int router_nsplit(int T, int H, int E, const double* part, size_t part_cap) {
    if (T < kRouterGemmMinTok || !part || part_cap < (size_t)T * E) return 0;
    const int tiles = ((T + kRgT - 1) / kRgT) * ((E + kRgE - 1) / kRgE);
    const int nk = H / kRgK;
    int nsplit = 1;
    for (int sp = 2; sp <= 64; ++sp)
        if (nk % sp == 0 && (size_t)sp * T * E <= part_cap && tiles * sp <= 2 * 148) nsplit = sp;
    return nsplit;
}

int router_kernel_count(int T, int H, int E, const double* part, size_t part_cap) {
    if (T == 0) return 0;
    return router_nsplit(T, H, E, part, part_cap) > 1 ? 2 : 1;
}

cudaError_t launch_router_logits(const float* wr, const float* bias, const void* x, coli_dtype dt, int T, int H, int E,
                                 double* logits, cudaStream_t st, double* part, size_t part_cap) {
    if (T == 0) return cudaSuccess;
    const int nsplit = router_nsplit(T, H, E, part, part_cap);
    if (nsplit > 0) {
        dim3 g((T + kRgT - 1) / kRgT, (E + kRgE - 1) / kRgE, nsplit);
        double* dst = nsplit == 1 ? logits : part;
        if (dt == COLI_F32)
            router_gemm_kernel<float><<<g, 128, 0, st>>>(wr, bias, (const float*)x, T, H, E, nsplit, dst);
        else
            router_gemm_kernel<__nv_bfloat16><<<g, 128, 0, st>>>(wr, bias, (const __nv_bfloat16*)x, T, H, E, nsplit, dst);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess || nsplit == 1) return e;
        const size_t n = (size_t)T * E;
        router_reduce_kernel<<<(int)((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048), 256, 0, st>>>(part, bias, T, E,
                                                                                                    nsplit, logits);
        return cudaGetLastError();
    }
    dim3 grid((E + 1) / 2, (T + kRouterTok - 1) / kRouterTok);
    if (dt == COLI_F32)
        router_logits_kernel<float><<<grid, 256, 0, st>>>(wr, bias, (const float*)x, T, H, E, logits);
    else
        router_logits_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(wr, bias, (const __nv_bfloat16*)x, T, H, E, logits);
    return cudaGetLastError();
}

cudaError_t launch_topk(const double* logits, int T, int E, int K, int32_t* ids, float* w, cudaStream_t st,
                        double topp, int e_lo, int e_hi) {
    if (T == 0) return cudaSuccess;
    if (e_hi < 0) e_hi = E;
    topk_kernel<<<(T + 7) / 8, 256, 0, st>>>(logits, T, E, K, topp, e_lo, e_hi, ids, w);
    return cudaGetLastError();
}

size_t plan_smem_bytes(int E) { return sizeof(int32_t) * ((size_t)kPlanWarps * E + E + 1); }

cudaError_t launch_plan(const int32_t* ids, int T, int K, int E, int S, const Plan& p, cudaStream_t st) {
    const size_t smem = plan_smem_bytes(E);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    plan_kernel<<<1, kPlanThreads, smem, st>>>(ids, T, K, E, S, p);
    return cudaGetLastError();
}

}  // namespace coli
