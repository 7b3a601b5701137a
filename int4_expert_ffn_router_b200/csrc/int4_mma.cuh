// int4_mma.cuh -- int4 x (few tokens) products on the tensor cores from
// register operands, for the decode kernel.
//
// A decode step multiplies each streamed weight by one to four tokens: the
// contraction is far too thin for shared-memory tensor-core tiles, but the
// CUDA-core instruction budget per streamed weight is the limit at HBM speed.
// Here the weights are the A operand of mma.m16n8k16 (16 weight rows x 16
// inputs per instruction) in their raw offset-binary fp16 form (one LOP3 per
// two weights, no per-weight arithmetic), the tokens the B operand as fp16
// hi + lo columns (about 22 significant bits after a per-token power-of-two
// scale), and the nibble offset is removed once per group through the
// accumulator's starting value.
#pragma once

#include "common.cuh"

namespace coli {

__device__ __forceinline__ uint32_t hfma2_u(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Weights as the A operand (16 rows x 16 inputs per mma), tokens as B: column
// n = 2j + p of B is part p (0 hi, 1 lo) of token j, so one instruction covers
// 256 weights for up to 4 tokens. The nibble offset is not removed per weight:
// the A fragments are the raw fp16 values 1024 + v (row gi) and 1024 + 16 v (row
// gi+8) of the offset-binary codes v = q + 8 (one logic op per pair), and the
// accumulators start at the group's offset correction
//     row gi:   -1032 * X,   row gi+8:  -1152 * X     (X = the column's sum of
// the group's 64 B values), so the MMAs return sum(q x) and 16 sum(q x).
// c = {row gi hi, row gi lo, row gi+8 hi, row gi+8 lo} corrections of token t.
// Steps 0, 2 and 1, 3 accumulate separately (two shorter dependency chains).
__device__ __forceinline__ void group_mma_aw_off(uint4 w, uint32_t sv, uint4 xb0, uint4 xb1, float4 c, float& acc0,
                                                 float& acc1) {
    float dd[2][4] = {{c.x, c.y, c.z, c.w}, {0.f, 0.f, 0.f, 0.f}};
    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
    const uint32_t bx[8] = {xb0.x, xb0.y, xb0.z, xb0.w, xb1.x, xb1.y, xb1.z, xb1.w};
    constexpr uint32_t MAGIC = 0x64006400u;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
        float* d = dd[s & 1];
        const uint32_t wv = words[s], ws = wv >> 8;
        const uint32_t r0 = lop3_and_or(wv, 0x000F000Fu, MAGIC);  // row gi,   k lo: 1024 + v
        const uint32_t r8 = lop3_and_or(wv, 0x00F000F0u, MAGIC);  // row gi+8, k lo: 1024 + 16 v
        const uint32_t r1 = lop3_and_or(ws, 0x000F000Fu, MAGIC);  // row gi,   k hi
        const uint32_t r9 = lop3_and_or(ws, 0x00F000F0u, MAGIC);  // row gi+8, k hi
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(r0), "r"(r8), "r"(r1), "r"(r9), "r"(bx[2 * s]), "r"(bx[2 * s + 1]));
    }
    float d[4] = {dd[0][0] + dd[1][0], dd[0][1] + dd[1][1], dd[0][2] + dd[1][2], dd[0][3] + dd[1][3]};
    const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sv));
    acc0 = fmaf(sc.x, d[0] + d[1], acc0);            // row gi: hi + lo columns of token t
    acc1 = fmaf(sc.y * 0.0625f, d[2] + d[3], acc1);  // row gi+8 (values carry a factor 16)
}

// Offset corrections for group_mma_aw_off from B fragments staged as in
// stage_bfrag: c[g * 4 + t] for token slot t < nt (zero otherwise), the
// column sums taken in a fixed order. xb: L = 8 * NT lanes per (g, half).
__device__ __forceinline__ void stage_offset_corr(const uint4* __restrict__ xb, float4* __restrict__ c, int G, int NT,
                                                  int nt, int tid, int nthr) {
    const int L = 8 * NT;
    for (int idx = tid; idx < G * 4; idx += nthr) {
        const int g = idx >> 2, t = idx & 3;
        float sum[2] = {0.0f, 0.0f};
        if (t < nt) {
#pragma unroll
            for (int part = 0; part < 2; ++part)
                for (int h = 0; h < 2; ++h)
                    for (int tt = 0; tt < 4; ++tt) {
                        const uint4 e = xb[(size_t)(2 * g + h) * L + 4 * (2 * t + part) + tt];
                        const uint32_t ev[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ev[q]));
                            sum[part] += f.x + f.y;
                        }
                    }
        }
        c[idx] = make_float4(-1032.0f * sum[0], -1032.0f * sum[1], -1152.0f * sum[0], -1152.0f * sum[1]);
    }
}

// 2^k as a float for k in [-126, 127].
__device__ __forceinline__ float exp2i(int k) { return __uint_as_float((uint32_t)(127 + k) << 23); }

template <typename XT>
__device__ __forceinline__ float load_in(const XT* p, bool coherent);
template <>
__device__ __forceinline__ float load_in<float>(const float* p, bool coherent) { return coherent ? __ldcg(p) : __ldg(p); }
template <>
__device__ __forceinline__ float load_in<__nv_bfloat16>(const __nv_bfloat16* p, bool coherent) {
    return __bfloat162float(*p);
}

__device__ __forceinline__ uint32_t split_pair(float a, float b, uint32_t& lo) {
    const __half ha = __float2half_rn(a), hb = __float2half_rn(b);
    const __half la = __float2half_rn(a - __half2float(ha)), lb = __float2half_rn(b - __half2float(hb));
    lo = (uint32_t)__half_as_ushort(la) | ((uint32_t)__half_as_ushort(lb) << 16);
    return (uint32_t)__half_as_ushort(ha) | ((uint32_t)__half_as_ushort(hb) << 16);
}

// Stage nt (<= NT) rows as B fragments for group_mma_aw_off, scaled per row by a
// power of two so that the row's largest magnitude lies in [2^14, 2^15) and
// split into fp16 hi + lo (about 22 significant bits together). Entry
//   xb[(g*2 + h)*8*NT + lane], lane < 8*NT: column n = lane/4 (token n/2, part
//   n%2), t = lane%4, steps s = 2h, 2h+1: {b0(s), b1(s), b0(s+1), b1(s+1)},
//   b0(s) = pair (k, k+1), b1(s) = pair (k+8, k+9), k = 64g + 16s + 2t.
// Columns of tokens >= nt hold zeros.
template <typename XT, int NT>
__device__ __forceinline__ void stage_bfrag(uint4* __restrict__ xb, float* scale_out, const XT* __restrict__ in,
                                            const int* rows, int nt, int C, bool coherent, int tid, int nthr,
                                            int bar, float* red) {
    const int lane = tid & 31, warp = tid >> 5, nw = nthr >> 5;
    float m[NT];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
        m[j] = 0.0f;
        if (j < nt) {
            const XT* r = in + (size_t)rows[j] * C;
            for (int c = tid; c < C; c += nthr) m[j] = fmaxf(m[j], fabsf(load_in<XT>(r + c, coherent)));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m[j] = fmaxf(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
        if (lane == 0) red[warp * NT + j] = m[j];
    }
    named_bar(bar, nthr);
    if (tid < NT) {
        float mx = 0.0f;
        for (int w = 0; w < nw; ++w) mx = fmaxf(mx, red[w * NT + tid]);
        int k = 0;
        const uint32_t eb = (__float_as_uint(mx) >> 23) & 0xFF;
        if (eb != 0 && eb != 0xFF) {
            k = 14 - ((int)eb - 127);
            k = k < -126 ? -126 : (k > 126 ? 126 : k);
        }
        red[nw * NT + tid] = exp2i(k);
        scale_out[tid] = exp2i(-k);
    }
    named_bar(bar, nthr);
    const int G = C / kGroup, L = 8 * NT;
    for (int idx = tid; idx < G * 2 * L; idx += nthr) {
        const int l = idx % L, gh = idx / L;
        const int g = gh >> 1, h = gh & 1;
        const int n = l >> 2, t = l & 3, j = n >> 1, part = n & 1;
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (j < nt) {
            const XT* src = in + (size_t)rows[j] * C;
            const float f = red[nw * NT + j];
            uint32_t outw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // q: (s = 2h + q/2, which = q%2 -> k offset 0 or 8)
                const int s = 2 * h + (q >> 1);
                const int k = g * 64 + s * 16 + 2 * t + ((q & 1) ? 8 : 0);
                uint32_t lo;
                const uint32_t hi = split_pair(load_in<XT>(src + k, coherent) * f, load_in<XT>(src + k + 1, coherent) * f, lo);
                outw[q] = part ? lo : hi;
            }
            o = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
        xb[(size_t)gh * L + l] = o;
    }
}

}  // namespace coli
