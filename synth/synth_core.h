/*
 * synth_core.h -- seeded, integer-exact synthetic input generator.
 *
 * This module produces the inputs that BOTH the CPU oracle and the CUDA path
 * consume: router weights, routed/shared expert weights already encoded in the
 * int4 group-of-64 container, activations, and the Zipf router bias. It holds
 * none of the MoE layer's arithmetic (no router product, no top-k, no expert
 * FFN, no combine). The same definitions compile for the host (gcc) and for
 * the device (nvcc), so that a layer can be generated directly in HBM and be
 * byte-identical to the host copy the oracle reads.
 *
 * Random source: the splitmix64 output function (Steele, Lea & Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014; constants as
 * published in Vigna's reference splitmix64.c) evaluated on a counter, so any
 * element can be drawn independently of the others.
 *
 * Approximate N(0,1): Irwin-Hall sum of twelve uniform 16-bit integers,
 *   z = (S - 393210) / 65536,  S = sum of the 12 draws.
 * S - 393210 is an integer below 2^20 in magnitude, so z is exact in fp32.
 * Mean 0, variance (65536^2 - 1)/65536^2 ~= 1, tails bounded at +-6.
 *
 * Weight encoding (the int4 gs64 container of the Colibri pages: "int4, group
 * size 64", with fp16 absmax/7 scales):
 *   per group of 64 consecutive elements along a row (the input dimension):
 *     s32 = absmax / 7 (fp32, IEEE division), s = fp16_rne(s32),
 *     q   = clamp(rint(w / s), -8, 7) (round half to even), q = 0 if s == 0.
 *   Canonical storage: byte j of a row holds elements 2j (low nibble) and
 *   2j+1 (high nibble), two's complement.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>
#include <math.h>
#include <string.h>

#ifdef __CUDACC__
#define SYNTH_FN __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ull

/* Tensor identifiers inside a stream key. */
enum {
    SYNTH_T_ROUTER = 1,   /* router weight [E][H]                   */
    SYNTH_T_EXPERT = 2,   /* expert matrix (expert id, matrix id)   */
    SYNTH_T_X      = 3,   /* activations for one step               */
    SYNTH_T_PERM   = 4    /* Zipf popularity permutation            */
};
/* Matrix ids inside an expert. gate [I][H], up [I][H], down [H][I]. */
enum { SYNTH_M_GATE = 0, SYNTH_M_UP = 1, SYNTH_M_DOWN = 2 };

SYNTH_FN uint64_t synth_fin64(uint64_t z)
{
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* Key of one tensor stream. */
SYNTH_FN uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t tensor,
                            uint32_t expert, uint32_t matrix)
{
    uint64_t id = ((uint64_t)(layer & 0xFFFFu) << 48) | ((uint64_t)(tensor & 0xFFu) << 40) |
                  ((uint64_t)(expert & 0xFFFFFFu) << 16) | (uint64_t)(matrix & 0xFFFFu);
    return synth_fin64(synth_fin64(seed + SYNTH_GAMMA) ^ (id + SYNTH_GAMMA));
}

/* n-th 64-bit draw of a stream: the splitmix64 output at state key + (n+1)*gamma. */
SYNTH_FN uint64_t synth_draw(uint64_t key, uint64_t n)
{
    return synth_fin64(key + (n + 1u) * SYNTH_GAMMA);
}

/* Integer Irwin-Hall offset S - 393210 for element i (three 64-bit draws). */
SYNTH_FN int32_t synth_ih(uint64_t key, uint64_t i)
{
    uint32_t s = 0;
    for (int k = 0; k < 3; ++k) {
        uint64_t r = synth_draw(key, 3u * i + (uint64_t)k);
        s += (uint32_t)(r & 0xFFFFu) + (uint32_t)((r >> 16) & 0xFFFFu) +
             (uint32_t)((r >> 32) & 0xFFFFu) + (uint32_t)(r >> 48);
    }
    return (int32_t)s - 393210;
}

SYNTH_FN uint32_t synth_f32_bits(float f)
{
#ifdef __CUDA_ARCH__
    return __float_as_uint(f);
#else
    uint32_t u; memcpy(&u, &f, 4); return u;
#endif
}

SYNTH_FN float synth_bits_f32(uint32_t u)
{
#ifdef __CUDA_ARCH__
    return __uint_as_float(u);
#else
    float f; memcpy(&f, &u, 4); return f;
#endif
}

/* Approximate standard normal, exact in fp32. */
SYNTH_FN float synth_gauss(uint64_t key, uint64_t i)
{
    return (float)synth_ih(key, i) * (1.0f / 65536.0f);
}

/* fp32 -> IEEE binary16, round to nearest even (NaN -> quiet NaN). */
SYNTH_FN uint16_t synth_f32_to_f16(float f)
{
    uint32_t x = synth_f32_bits(f);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t ax = x & 0x7FFFFFFFu;
    if (ax > 0x7F800000u) return (uint16_t)(sign | 0x7E00u);
    if (ax >= 0x47800000u) return (uint16_t)(sign | 0x7C00u); /* >= 65536 (and inf) */
    if (ax >= 0x38800000u) {                                  /* normal half range */
        uint32_t h = (ax - 0x38000000u) >> 13;                /* rebias 127 -> 15  */
        uint32_t rem = ax & 0x1FFFu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u; /* may round to inf */
        return (uint16_t)(sign | h);
    }
    /* subnormal half: value * 2^24 rounded to an integer in [0, 1024] */
    uint32_t e = ax >> 23;
    uint32_t m = (ax & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    if (e == 0) e = 1;
    uint32_t shift = 126u - e;
    if (shift >= 25u) return (uint16_t)sign;
    uint32_t r = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1u);
    if (rem > half || (rem == half && (r & 1u))) r += 1u;
    return (uint16_t)(sign | r);
}

/* IEEE binary16 -> fp32 (exact). */
SYNTH_FN float synth_f16_to_f32(uint16_t h)
{
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = ((uint32_t)h >> 10) & 0x1Fu;
    uint32_t m = (uint32_t)h & 0x3FFu;
    if (e == 0x1Fu) return synth_bits_f32(sign | 0x7F800000u | (m << 13));
    if (e != 0) return synth_bits_f32(sign | ((e + 112u) << 23) | (m << 13));
    if (m == 0) return synth_bits_f32(sign);
    /* subnormal: m * 2^-24 */
    float v = (float)m * (1.0f / 16777216.0f);
    return (sign ? -v : v);
}

/* fp32 -> bfloat16 bits, round to nearest even (NaN stays NaN). */
SYNTH_FN uint16_t synth_f32_to_bf16(float f)
{
    uint32_t x = synth_f32_bits(f);
    if ((x & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((x >> 16) | 0x40u);
    uint32_t lsb = (x >> 16) & 1u;
    x += 0x7FFFu + lsb;
    return (uint16_t)(x >> 16);
}

#ifdef __CUDA_ARCH__
#define SYNTH_DIV(a, b) __fdiv_rn((a), (b))
#define SYNTH_MUL(a, b) __fmul_rn((a), (b))
#else
#define SYNTH_DIV(a, b) ((a) / (b))
#define SYNTH_MUL(a, b) ((a) * (b))
#endif

/*
 * Encode one group of 64 weights of an expert matrix with `cols` columns:
 * element (r, 64g + i) is wscale * gauss(key, r*cols + 64g + i). The group is
 * generated twice (once for its absmax, once to encode), so no 64-element
 * array is needed on the device. Writes 32 canonical bytes and the fp16 scale.
 */
SYNTH_FN void synth_weight_group(uint64_t key, int cols, int r, int g, float wscale,
                                 uint8_t* qbytes /*32*/, uint16_t* scale)
{
    uint64_t base = (uint64_t)r * (uint64_t)cols + (uint64_t)g * 64u;
    float amax = 0.0f;
    for (int i = 0; i < 64; ++i) {
        float a = fabsf(SYNTH_MUL(wscale, synth_gauss(key, base + (uint64_t)i)));
        amax = a > amax ? a : amax;
    }
    uint16_t s16 = synth_f32_to_f16(SYNTH_DIV(amax, 7.0f));
    float s = synth_f16_to_f32(s16);
    *scale = s16;
    for (int j = 0; j < 32; ++j) {
        uint32_t nib[2];
        for (int h = 0; h < 2; ++h) {
            float w = SYNTH_MUL(wscale, synth_gauss(key, base + (uint64_t)(2 * j + h)));
            int v = 0;
            if (s > 0.0f) {
                float q = rintf(SYNTH_DIV(w, s));
                q = q < -8.0f ? -8.0f : (q > 7.0f ? 7.0f : q);
                v = (int)q;
            }
            nib[h] = (uint32_t)v & 0x0Fu;
        }
        qbytes[j] = (uint8_t)(nib[0] | (nib[1] << 4));
    }
}

#endif /* SYNTH_CORE_H */
