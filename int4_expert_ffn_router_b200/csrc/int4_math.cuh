// int4_math.cuh -- the in-register int4 -> fp32 dequantisation and the
// packed-FFMA2 dot products shared by the CUDA-core expert kernels.
#pragma once

#include "common.cuh"

namespace coli {

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 as_f2(uint32_t lo_bits, uint32_t hi_bits) {
    return make_float2(__uint_as_float(lo_bits), __uint_as_float(hi_bits));
}

// Codes of one 32-bit word (layout in common.cuh) as four float pairs:
// p04 = (row gi: col a, col a+1), p26 = (row gi: col a+8, a+9),
// p15 = (row gi+8: col a, a+1),   p37 = (row gi+8: col a+8, a+9).
__device__ __forceinline__ void decode_word(uint32_t w, float2& p04, float2& p26, float2& p15, float2& p37) {
    constexpr uint32_t M = 0x4B000000u;  // 2^23
    const uint32_t wh = w >> 12;
    float2 f04 = as_f2(lop3_and_or(w, 0x0000000Fu, M), lop3_and_or(w, 0x000F0000u, M));
    float2 f15 = as_f2(lop3_and_or(w, 0x000000F0u, M), lop3_and_or(wh, 0x00000F00u, M));
    float2 f26 = as_f2(lop3_and_or(w, 0x00000F00u, M), lop3_and_or(wh, 0x0000F000u, M));
    float2 f37 = as_f2(lop3_and_or(w, 0x0000F000u, M), lop3_and_or(wh, 0x000F0000u, M));
    // f = 2^23 + v * 2^k  ->  q = f * 2^-k - (2^(23-k) + 8): exact
    p04 = ffma2(f04, make_float2(1.0f, 0x1p-16f), make_float2(-8388616.0f, -136.0f));
    p15 = ffma2(f15, make_float2(0x1p-4f, 0x1p-8f), make_float2(-524296.0f, -32776.0f));
    p26 = ffma2(f26, make_float2(0x1p-8f, 0x1p-12f), make_float2(-32776.0f, -2056.0f));
    p37 = ffma2(f37, make_float2(0x1p-12f, 0x1p-16f), make_float2(-2056.0f, -136.0f));
}

template <typename XT>
__device__ __forceinline__ float to_f32(XT v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Stage rows of the input (C inputs each) into shared memory in lane order:
// xs[tb][g][ti][s] = float4(x[c], x[c+1], x[c+8], x[c+9]), c = 64g + 16s + 2ti,
// using threads tid = 0..nthreads-1. `coherent` reads through L2 only (for
// data written earlier by other CTAs of the same kernel).
template <typename XT, bool coherent = false>
__device__ __forceinline__ void stage_rows(float4* xs, const XT* __restrict__ in, const int32_t* rows, int nt, int C,
                                           int tid, int nthreads) {
    const int G = C / kGroup;
    for (int idx = tid; idx < nt * G * 16; idx += nthreads) {
        int tb = idx / (G * 16);
        int r = idx - tb * G * 16;
        int g = r >> 4, ti = (r >> 2) & 3, s = r & 3;
        int c = g * 64 + s * 16 + ti * 2;
        const XT* src = in + (size_t)rows[tb] * C + c;
        float v0, v1, v8, v9;
        if constexpr (coherent && sizeof(XT) == 4) {
            const float2 a = __ldcg(reinterpret_cast<const float2*>(src));
            const float2 b = __ldcg(reinterpret_cast<const float2*>(src + 8));
            v0 = a.x; v1 = a.y; v8 = b.x; v9 = b.y;
        } else {
            v0 = to_f32<XT>(src[0]); v1 = to_f32<XT>(src[1]); v8 = to_f32<XT>(src[8]); v9 = to_f32<XT>(src[9]);
        }
        xs[((tb * G + g) * 4 + ti) * 4 + s] = make_float4(v0, v1, v8, v9);
    }
}

// One 64-input group of a 16-row sub-tile against nt <= NT staged inputs.
// `w` is this lane's 16 bytes of the group (layout in common.cuh), `sv` the
// lane's fp16 scale pair (row gi, row gi+8), `xg` the staged inputs of group g
// (xs + g*16 for token 0; token stride `tstride` float4). Accumulates into
// acc0 (row gi) and acc1 (row gi+8).
template <int NT>
__device__ __forceinline__ void group_dot(uint4 w, uint32_t sv, const float4* xg, int tstride, int ti, int nt,
                                          float acc0[NT], float acc1[NT]) {
    const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sv));
    float2 a0[NT], a1[NT];
#pragma unroll
    for (int tb = 0; tb < NT; ++tb) { a0[tb] = make_float2(0.f, 0.f); a1[tb] = make_float2(0.f, 0.f); }
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        float2 p04, p26, p15, p37;
        decode_word(words[s], p04, p26, p15, p37);
#pragma unroll
        for (int tb = 0; tb < NT; ++tb) {
            if (tb < nt) {
                const float4 xv = xg[tb * tstride + ti * 4 + s];
                const float2 x01 = make_float2(xv.x, xv.y), x89 = make_float2(xv.z, xv.w);
                a0[tb] = ffma2(p04, x01, a0[tb]);
                a0[tb] = ffma2(p26, x89, a0[tb]);
                a1[tb] = ffma2(p15, x01, a1[tb]);
                a1[tb] = ffma2(p37, x89, a1[tb]);
            }
        }
    }
#pragma unroll
    for (int tb = 0; tb < NT; ++tb) {
        if (tb < nt) {
            acc0[tb] = fmaf(sc.x, a0[tb].x + a0[tb].y, acc0[tb]);
            acc1[tb] = fmaf(sc.y, a1[tb].x + a1[tb].y, acc1[tb]);
        }
    }
}

}  // namespace coli
