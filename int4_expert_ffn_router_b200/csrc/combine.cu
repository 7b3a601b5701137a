// combine.cu -- routing-weighted combine of the expert outputs, and the
// RMSNorm of the residual stack.
#include "common.cuh"
#include "kernels.cuh"

namespace coli {

// y[t][c] = residual[t][c] + sum_j o[TK + jT + t][c] + sum_k w[t][k] o[pos[t][k]][c]
// Shared experts (weight 1, part of the always-on dense block: "Colibri: 2400
// lines of pure C ...", kechuai.cn, section 一) first, then the routed experts
// in routing order; fixed order, so the result is deterministic.
template <typename YT>
__global__ void combine_kernel(const float* __restrict__ o, Plan p, int T, int H, int K, int S,
                               const float* __restrict__ residual, YT* __restrict__ y) {
    // one thread per (token, 4 columns); a grid-stride loop covers any T
    const int H4 = H / 4;
    const size_t n = (size_t)T * H4;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / H4), c4 = (int)(i % H4);
        float4 acc = residual ? reinterpret_cast<const float4*>(residual + (size_t)t * H)[c4] : make_float4(0, 0, 0, 0);
        for (int j = 0; j < S; ++j) {
            const float4 v = reinterpret_cast<const float4*>(o + (size_t)(T * K + j * T + t) * H)[c4];
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        for (int k = 0; k < K; ++k) {
            const int q = p.pos[t * K + k];
            if (q < 0) continue;  // an empty slot (expert of another rank)
            const float wk = p.w[t * K + k];
            const float4 v = reinterpret_cast<const float4*>(o + (size_t)q * H)[c4];
            acc.x = fmaf(wk, v.x, acc.x);
            acc.y = fmaf(wk, v.y, acc.y);
            acc.z = fmaf(wk, v.z, acc.z);
            acc.w = fmaf(wk, v.w, acc.w);
        }
        if constexpr (sizeof(YT) == 4) {
            reinterpret_cast<float4*>(y + (size_t)t * H)[c4] = acc;
        } else {
            __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&lo);
            u.y = *reinterpret_cast<uint32_t*>(&hi);
            reinterpret_cast<uint2*>(y + (size_t)t * H)[c4] = u;
        }
    }
}

cudaError_t launch_combine(const float* o, const Plan& p, int T, int H, int K, int S, const float* residual, void* y,
                           coli_dtype ydt, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const size_t blocks = ((size_t)T * (H / 4) + 127) / 128;
    const int grid = (int)(blocks < 148 * 32 ? blocks : 148 * 32);
    if (ydt == COLI_F32)
        combine_kernel<float><<<grid, 128, 0, st>>>(o, p, T, H, K, S, residual, (float*)y);
    else
        combine_kernel<__nv_bfloat16><<<grid, 128, 0, st>>>(o, p, T, H, K, S, residual, (__nv_bfloat16*)y);
    return cudaGetLastError();
}

// RMSNorm with unit gain; the sum of squares and the reciprocal root in fp64.
__global__ void rmsnorm_kernel(const float* __restrict__ x, int H, float eps, float* __restrict__ out) {
    __shared__ double red[32];
    const int t = blockIdx.x;
    const float* xr = x + (size_t)t * H;
    double ss = 0.0;
    for (int c = threadIdx.x; c < H; c += blockDim.x) ss += (double)xr[c] * (double)xr[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (threadIdx.x == 0) red[0] = 1.0 / sqrt(v / (double)H + (double)eps);
    }
    __syncthreads();
    const double r = red[0];
    for (int c = threadIdx.x; c < H; c += blockDim.x) out[(size_t)t * H + c] = (float)((double)xr[c] * r);
}

cudaError_t launch_rmsnorm(const float* x, int T, int H, float eps, float* out, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    rmsnorm_kernel<<<T, 256, 0, st>>>(x, H, eps, out);
    return cudaGetLastError();
}

}  // namespace coli
