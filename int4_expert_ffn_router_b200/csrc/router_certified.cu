// router_certified.cu -- the router of token batches in fp32 with a certified
// selection, recomputing in fp64 only what the selection cannot settle.
//
// The router and its top-K are those of router.cu (fp64 logits, K largest,
// equal logits to the lower id, softmax over the K): "Colibri: 2400 lines of
// pure C ..." (kechuai.cn), section 一. The fp64 GEMM of a 2048-token batch
// is bound by the FP64 rate; this form computes the logits in fp32 with a
// known summation order and a rigorous error bound per logit, and the set of
// the K largest logits is taken from the fp32 values only when the bound
// proves it is the set of the exact logits:
//   |v_e - l_e| <= eps_e = c * ||Wr_e||_2 * ||x_t||_2   (c from the order)
//   min over the selected (v - eps) > max over the others (v + eps)
// => every selected exact logit exceeds every other one, so the selection of
// the exact (and of any fp64) logits is the same set. The order within the
// set and the weights then come from the K selected logits recomputed in
// fp64. A token whose bound does not separate the set (a near tie at the
// K-th place) gets all of its logits in fp64 and the fp64 top-K.
#include "common.cuh"
#include "kernels.cuh"
#include "topk.cuh"

namespace coli {
namespace {

// fp32 GEMM: CTA tile 64 tokens x 128 experts x one of kCfSplit ranges of
// the input dimension, 256 threads; thread (ty, tx) owns tokens 8ty..8ty+7
// and experts 4tx..4tx+3. Each output sums kCfBlk inputs at a time by
// sequential FMAs from 0 into `part`, then adds `part` to `tot`; the
// kCfSplit range sums are added in fp64 by the certify kernel. The error of a
// logit is at most
//   (gamma_kCfBlk + gamma_(blocks per range - 1) (1 + gamma_kCfBlk)) * sum |w x|
// (plus the fp64 additions, far below).
constexpr int kCfT = 64, kCfE = 128, kCfK = 16, kCfBlk = 128, kCfSplit = 4, kCfThreads = 256;

template <typename XT>
__device__ __forceinline__ void cf_load8(const XT* p, float v[8]);
template <>
__device__ __forceinline__ void cf_load8<float>(const float* p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void cf_load8<__nv_bfloat16>(const __nv_bfloat16* p, float v[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

template <typename XT>
__global__ void __launch_bounds__(kCfThreads, 2) router_f32_kernel(const float* __restrict__ wr, const XT* __restrict__ x,
                                                            int T, int H, int E, float* __restrict__ l32) {
    __shared__ __align__(16) float xs[2][kCfK][kCfT];  // 8 KB, k-major
    __shared__ __align__(16) float ws[2][kCfK][kCfE];  // 16 KB, k-major
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
    const int t0 = blockIdx.x * kCfT, e0 = blockIdx.y * kCfE;
    const int hspan = H / kCfSplit, h0 = blockIdx.z * hspan;
    // loaders: x row tid / 4, inputs 4 (tid & 3) .. +3; Wr row tid / 2, inputs 8 (tid & 1) .. +7
    const int xr = tid >> 2, xk = (tid & 3) * 4, wrow = tid >> 1, wk = (tid & 1) * 8;
    const bool xok = t0 + xr < T, wok = e0 + wrow < E;
    const XT* xp = x + (size_t)(xok ? t0 + xr : 0) * H + h0 + xk;
    const float* wp = wr + (size_t)(wok ? e0 + wrow : 0) * H + h0 + wk;
    float xv[4], wv[8];
    auto fetch = [&](int k0) {
        if (xok) {
            if constexpr (sizeof(XT) == 4) {
                const float4 f = *reinterpret_cast<const float4*>(xp + k0);
                xv[0] = f.x; xv[1] = f.y; xv[2] = f.z; xv[3] = f.w;
            } else {
                const uint2 u = *reinterpret_cast<const uint2*>(xp + k0);
                xv[0] = __uint_as_float(u.x << 16); xv[1] = __uint_as_float(u.x & 0xFFFF0000u);
                xv[2] = __uint_as_float(u.y << 16); xv[3] = __uint_as_float(u.y & 0xFFFF0000u);
            }
        } else {
            xv[0] = xv[1] = xv[2] = xv[3] = 0.0f;
        }
        if (wok) {
            cf_load8<float>(wp + k0, wv);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) wv[i] = 0.0f;
        }
    };
    auto stash = [&](int b) {
#pragma unroll
        for (int i = 0; i < 4; ++i) xs[b][xk + i][xr] = xv[i];
#pragma unroll
        for (int i = 0; i < 8; ++i) ws[b][wk + i][wrow] = wv[i];
    };
    float part[8][4], tot[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = tot[i][j] = 0.0f;
    const int nk = hspan / kCfK;
    fetch(0);
    stash(0);
    __syncthreads();
    for (int c = 0; c < nk; ++c) {
        const int b = c & 1;
        if (c + 1 < nk) fetch((c + 1) * kCfK);
#pragma unroll
        for (int k = 0; k < kCfK; ++k) {
            const float4 xa = *reinterpret_cast<const float4*>(&xs[b][k][8 * ty]);
            const float4 xb = *reinterpret_cast<const float4*>(&xs[b][k][8 * ty + 4]);
            const float4 wa = *reinterpret_cast<const float4*>(&ws[b][k][4 * tx]);
            const float xq[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
            const float wq[4] = {wa.x, wa.y, wa.z, wa.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) part[i][j] = fmaf(wq[j], xq[i], part[i][j]);
        }
        if (((c + 1) * kCfK) % kCfBlk == 0 || c + 1 == nk) {  // end of a summation block
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    tot[i][j] += part[i][j];
                    part[i][j] = 0.0f;
                }
        }
        if (c + 1 < nk) {
            stash(b ^ 1);
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + 8 * ty + i;
        if (t >= T) continue;
        const int e = e0 + 4 * tx;
        float* dst = l32 + ((size_t)blockIdx.z * T + t) * E + e;
        if (e + 3 < E) *reinterpret_cast<float4*>(dst) = make_float4(tot[i][0], tot[i][1], tot[i][2], tot[i][3]);
        else
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (e + j < E) dst[j] = tot[i][j];
    }
}

// ||Wr_e||_2, rounded up (fp64 sum of squares, square root, one ulp up).
__global__ void router_norm_kernel(const float* __restrict__ wr, int H, int E, double* __restrict__ wn) {
    const int e = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (e >= E) return;
    double s = 0.0;
    for (int h = lane; h < H; h += 32) s = fma((double)wr[(size_t)e * H + h], (double)wr[(size_t)e * H + h], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wn[e] = sqrt(s) * (1.0 + 1e-14);
}

// One warp per token: the K largest of the fp32 logits (plus bias, in fp64),
// the certificate, then either the K logits in fp64 with their order and
// weights, or the token on the list of tokens for the fp64 fallback.
// ||x_t||_2 in fp64, rounded up, one warp per token.
template <typename XT>
__global__ void __launch_bounds__(256) token_norm_kernel(const XT* __restrict__ x, int T, int H, double* __restrict__ xn) {
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (t >= T) return;
    double ss = 0.0;
    for (int h = 8 * lane; h < H; h += 256) {
        float v[8];
        cf_load8<XT>(x + (size_t)t * H + h, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) ss = fma((double)v[i], (double)v[i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (lane == 0) xn[t] = sqrt(ss) * (1.0 + 1e-14);
}

template <typename XT>
__global__ void __launch_bounds__(256) router_certify_kernel(const float* __restrict__ l32, const double* __restrict__ wn,
                                                             const double* __restrict__ xnorm,
                                                             const float* __restrict__ wr, const float* __restrict__ bias,
                                                             const XT* __restrict__ x, int T, int H, int E, int K,
                                                             double c_bound, double topp, int e_lo, int e_hi,
                                                             int32_t* __restrict__ ids, float* __restrict__ w,
                                                             int* __restrict__ fail) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const XT* xrow = x + (size_t)t * H;
    const double xn = xnorm[t];
    // this lane's experts lane + 32 i (i < 8): value and bound
    unsigned long long k8[8];
    int id8[8];
    double lo8[8], hi8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        k8[i] = 0ull;
        id8[i] = 0x7fffffff;
        lo8[i] = hi8[i] = 0.0;
        if (e < E) {
            double v = (double)bias[e];
#pragma unroll
            for (int z = 0; z < kCfSplit; ++z) v += (double)l32[((size_t)z * T + t) * E + e];
            const double eps = c_bound * wn[e] * xn * (1.0 + 1e-12) + fabs(v) * 4.5e-16 + 1e-300;
            k8[i] = order_key(v);
            id8[i] = e;
            lo8[i] = v - eps;
            hi8[i] = v + eps;
        }
    }
    // the K largest values (descending, equal values to the lower id): each lane sorts its
    // 8 entries, then K rounds take the warp's best head
    unsigned long long ks[8];
    int is[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { ks[i] = k8[i]; is[i] = id8[i]; }
    cx8(ks, is, 0, 1); cx8(ks, is, 2, 3); cx8(ks, is, 4, 5); cx8(ks, is, 6, 7);
    cx8(ks, is, 0, 2); cx8(ks, is, 1, 3); cx8(ks, is, 4, 6); cx8(ks, is, 5, 7);
    cx8(ks, is, 1, 2); cx8(ks, is, 5, 6);
    cx8(ks, is, 0, 4); cx8(ks, is, 1, 5); cx8(ks, is, 2, 6); cx8(ks, is, 3, 7);
    cx8(ks, is, 2, 4); cx8(ks, is, 3, 5);
    cx8(ks, is, 1, 2); cx8(ks, is, 3, 4); cx8(ks, is, 5, 6);
    int my_id = -1;
    unsigned selmask = 0u;  // which of this lane's entries were selected (expert lane + 32 i: bit i)
    for (int r = 0; r < K; ++r) {
        const unsigned khi = (unsigned)(ks[0] >> 32), klo = (unsigned)ks[0];
        const unsigned bhi = __reduce_max_sync(0xffffffffu, khi);
        const unsigned blo = __reduce_max_sync(0xffffffffu, khi == bhi ? klo : 0u);
        const bool holds = khi == bhi && klo == blo;
        const int bi = (int)__reduce_min_sync(0xffffffffu, holds ? (unsigned)is[0] : 0x7fffffffu);
        if (holds && is[0] == bi) {
            selmask |= 1u << ((bi - lane) >> 5);
#pragma unroll
            for (int i = 0; i < 7; ++i) { ks[i] = ks[i + 1]; is[i] = is[i + 1]; }
            ks[7] = 0ull;
            is[7] = 0x7fffffff;
        }
        if (lane == r) my_id = bi;
    }
    // certificate: every selected lower bound above every other upper bound
    double sel_lo = 1e300, oth_hi = -1e300;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (id8[i] == 0x7fffffff) continue;
        if ((selmask >> i) & 1u) sel_lo = fmin(sel_lo, lo8[i]);
        else oth_hi = fmax(oth_hi, hi8[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sel_lo = fmin(sel_lo, __shfl_xor_sync(0xffffffffu, sel_lo, o));
        oth_hi = fmax(oth_hi, __shfl_xor_sync(0xffffffffu, oth_hi, o));
    }
    if (!(sel_lo > oth_hi)) {  // not separated: every logit of this token in fp64 (fallback kernels)
        if (lane == 0) fail[1 + atomicAdd(fail, 1)] = t;
        return;
    }
    // the selected logits in fp64, eight at a time by the whole warp: lane l sums inputs
    // 4l + 128 i (i = 0, 1, ...) of each, then a fixed xor tree
    double my_l = 0.0;
    for (int k0 = 0; k0 < K; k0 += 8) {
        int ek[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) ek[j] = __shfl_sync(0xffffffffu, my_id, (k0 + j) & 31);
        double sj[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int h = 4 * lane; h < H; h += 128) {
            float xv[4];
            if constexpr (sizeof(XT) == 4) {
                const float4 f = *reinterpret_cast<const float4*>(xrow + h);
                xv[0] = f.x; xv[1] = f.y; xv[2] = f.z; xv[3] = f.w;
            } else {
                const uint2 u = *reinterpret_cast<const uint2*>(xrow + h);
                xv[0] = __uint_as_float(u.x << 16); xv[1] = __uint_as_float(u.x & 0xFFFF0000u);
                xv[2] = __uint_as_float(u.y << 16); xv[3] = __uint_as_float(u.y & 0xFFFF0000u);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (k0 + j >= K) continue;
                const float4 w4 = *reinterpret_cast<const float4*>(wr + (size_t)ek[j] * H + h);
                sj[j] = fma((double)w4.x, (double)xv[0], sj[j]);
                sj[j] = fma((double)w4.y, (double)xv[1], sj[j]);
                sj[j] = fma((double)w4.z, (double)xv[2], sj[j]);
                sj[j] = fma((double)w4.w, (double)xv[3], sj[j]);
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sj[j] += __shfl_xor_sync(0xffffffffu, sj[j], o);
            if (lane == k0 + j && k0 + j < K) my_l = sj[j] + (double)bias[ek[j]];
        }
    }
    // order among the selected: rank by (fp64 logit descending, id ascending)
    const unsigned long long my_key = lane < K ? order_key(my_l) : 0ull;
    int rank = 0;
    for (int k = 0; k < K; ++k) {
        const unsigned long long ok = __shfl_sync(0xffffffffu, my_key, k);
        const int oi = __shfl_sync(0xffffffffu, my_id, k);
        rank += ok > my_key || (ok == my_key && oi < my_id);
    }
    // lane r takes the entry of rank r
    int src = 0;
    for (int k = 0; k < K; ++k) src = __shfl_sync(0xffffffffu, rank, k) == lane ? k : src;
    const unsigned long long skey = __shfl_sync(0xffffffffu, my_key, src);
    const int sid = __shfl_sync(0xffffffffu, my_id, src);
    const unsigned long long top = __shfl_sync(0xffffffffu, skey, 0);
    int id;
    float wt;
    topk_weights(lane < K ? skey : 0ull, top, lane < K ? sid : -1, K, topp, lane, &id, &wt);
    if (lane < K) {
        ids[(size_t)t * K + lane] = (id >= e_lo && id < e_hi) ? id : -1;
        w[(size_t)t * K + lane] = wt;
    }
}

// Fallback: fp64 logits of the listed tokens. CTA (bx, by): experts 2bx,
// 2bx+1 (four warps each, a quarter of H per warp) for listed tokens by,
// by + gridDim.y, ...
template <typename XT>
__global__ void __launch_bounds__(256) router_fallback_kernel(const float* __restrict__ wr, const float* __restrict__ bias,
                                                              const XT* __restrict__ x, int H, int E,
                                                              const int* __restrict__ fail, double* __restrict__ logits) {
    __shared__ double part[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 2 + (warp >> 2), quarter = warp & 3, seg = H / 4;
    const int n = *fail;
    for (int f = blockIdx.y; f < n; f += gridDim.y) {
        const int t = fail[1 + f];
        double s = 0.0;
        if (e < E) {
            const float* wrow = wr + (size_t)e * H + quarter * seg;
            const XT* xrow = x + (size_t)t * H + quarter * seg;
            for (int h = lane; h < seg; h += 32) {
                float v;
                if constexpr (sizeof(XT) == 4) v = xrow[h];
                else v = __bfloat162float(xrow[h]);
                s = fma((double)wrow[h], (double)v, s);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[warp] = s;
        __syncthreads();
        if (threadIdx.x < 2) {
            const int ee = blockIdx.x * 2 + threadIdx.x;
            if (ee < E) {
                const double* p = part + 4 * threadIdx.x;
                logits[(size_t)t * E + ee] = ((p[0] + p[1]) + p[2]) + p[3] + (double)bias[ee];
            }
        }
        __syncthreads();
    }
}

// Fallback top-K of the listed tokens, one warp per token.
__global__ void __launch_bounds__(256) router_fallback_topk_kernel(const double* __restrict__ logits, int E, int K,
                                                                   double topp, int e_lo, int e_hi,
                                                                   const int* __restrict__ fail,
                                                                   int32_t* __restrict__ ids, float* __restrict__ w) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = *fail;
    for (int f = blockIdx.x * 8 + warp; f < n; f += gridDim.x * 8) {
        const int t = fail[1 + f];
        int id;
        float wt;
        if (E <= 256) warp_topk8<true>(logits + (size_t)t * E, E, K, topp, lane, &id, &wt);
        else warp_topk<true>(logits + (size_t)t * E, E, K, topp, lane, &id, &wt);
        if (lane < K) {
            ids[(size_t)t * K + lane] = (id >= e_lo && id < e_hi) ? id : -1;
            w[(size_t)t * K + lane] = wt;
        }
    }
}

double gamma_n(int n) {
    const double u = 1.0 / 16777216.0;  // 2^-24
    return n * u / (1.0 - n * u);
}

}  // namespace

bool router_certified_supported(int H, int E) { return H % (kCfSplit * kCfBlk) == 0 && E <= 256; }

cudaError_t launch_router_norms(const float* wr, int H, int E, double* wn, cudaStream_t st) {
    router_norm_kernel<<<(E + 7) / 8, 256, 0, st>>>(wr, H, E, wn);
    return cudaGetLastError();
}

cudaError_t launch_router_certified(const float* wr, const double* wn, const float* bias, const void* x, coli_dtype dt,
                                    int T, int H, int E, int K, double topp, int e_lo, int e_hi, float* l32,
                                    double* xnorm, int* fail, double* logits, int32_t* ids, float* w, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (e_hi < 0) e_hi = E;
    const int nb = H / kCfSplit / kCfBlk;  // summation blocks per range
    // fp32 sums, plus the fp64 additions of the ranges and the bias
    const double c = gamma_n(kCfBlk) + gamma_n(nb - 1) * (1.0 + gamma_n(kCfBlk)) + 1e-15;
    cudaError_t e = cudaMemsetAsync(fail, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    dim3 g((T + kCfT - 1) / kCfT, (E + kCfE - 1) / kCfE, kCfSplit);
    if (dt == COLI_F32) router_f32_kernel<float><<<g, kCfThreads, 0, st>>>(wr, (const float*)x, T, H, E, l32);
    else router_f32_kernel<__nv_bfloat16><<<g, kCfThreads, 0, st>>>(wr, (const __nv_bfloat16*)x, T, H, E, l32);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dt == COLI_F32) token_norm_kernel<float><<<(T + 7) / 8, 256, 0, st>>>((const float*)x, T, H, xnorm);
    else token_norm_kernel<__nv_bfloat16><<<(T + 7) / 8, 256, 0, st>>>((const __nv_bfloat16*)x, T, H, xnorm);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dt == COLI_F32)
        router_certify_kernel<float><<<(T + 7) / 8, 256, 0, st>>>(l32, wn, xnorm, wr, bias, (const float*)x, T, H, E, K,
                                                                  c, topp, e_lo, e_hi, ids, w, fail);
    else
        router_certify_kernel<__nv_bfloat16><<<(T + 7) / 8, 256, 0, st>>>(l32, wn, xnorm, wr, bias,
                                                                          (const __nv_bfloat16*)x, T, H, E, K, c, topp,
                                                                          e_lo, e_hi, ids, w, fail);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dim3 gf((E + 1) / 2, 64);
    if (dt == COLI_F32) router_fallback_kernel<float><<<gf, 256, 0, st>>>(wr, bias, (const float*)x, H, E, fail, logits);
    else router_fallback_kernel<__nv_bfloat16><<<gf, 256, 0, st>>>(wr, bias, (const __nv_bfloat16*)x, H, E, fail, logits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    router_fallback_topk_kernel<<<16, 256, 0, st>>>(logits, E, K, topp, e_lo, e_hi, fail, ids, w);
    return cudaGetLastError();
}

}  // namespace coli
