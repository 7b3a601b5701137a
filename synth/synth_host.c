/*
 * synth_host.c -- host side of the seeded synthetic input generator
 * (definitions in synth_core.h). Test and benchmark infrastructure: it builds
 * inputs, it computes nothing of the MoE layer.
 *
 * Canonical expert buffer (what coli_moe_layer_create and the oracle read):
 *   q: gate [I][H/2] | up [I][H/2] | down [H][I/2]  bytes, low nibble = even element
 *   s: gate [I][H/64] | up [I][H/64] | down [H][I/64]  fp16 bits
 */
#include "synth_core.h"

#include <stdlib.h>
#include <math.h>

#define SYNTH_API __attribute__((visibility("default")))

/* One matrix [rows][cols] of expert `expert` into canonical storage. */
static void gen_matrix(uint64_t seed, int layer, int expert, int matrix, int rows, int cols,
                       float wscale, uint8_t* q, uint16_t* s)
{
    uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_EXPERT, (uint32_t)expert, (uint32_t)matrix);
    int groups = cols / 64;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r)
        for (int g = 0; g < groups; ++g)
            synth_weight_group(key, cols, r, g, wscale, q + (size_t)r * (cols / 2) + (size_t)g * 32,
                               s + (size_t)r * groups + g);
}

SYNTH_API int synth_expert(uint64_t seed, int layer, int expert, int H, int I, float wscale,
                           uint8_t* q, uint16_t* s)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64 || !q || !s) return -1;
    size_t gq = (size_t)I * H / 2, gs = (size_t)I * H / 64;
    gen_matrix(seed, layer, expert, SYNTH_M_GATE, I, H, wscale, q, s);
    gen_matrix(seed, layer, expert, SYNTH_M_UP, I, H, wscale, q + gq, s + gs);
    gen_matrix(seed, layer, expert, SYNTH_M_DOWN, H, I, wscale, q + 2 * gq, s + 2 * gs);
    return 0;
}

/* Unencoded fp32 weights of one matrix (used to pin the encoder's round trip). */
SYNTH_API int synth_matrix_f32(uint64_t seed, int layer, int expert, int matrix, int rows, int cols,
                               float wscale, float* w)
{
    if (rows <= 0 || cols <= 0 || !w) return -1;
    uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_EXPERT, (uint32_t)expert, (uint32_t)matrix);
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r)
        for (int c = 0; c < cols; ++c)
            w[(size_t)r * cols + c] =
                SYNTH_MUL(wscale, synth_gauss(key, (uint64_t)r * (uint64_t)cols + (uint64_t)c));
    return 0;
}

/* Encode an arbitrary fp32 matrix [rows][cols] (cols % 64 == 0) into the container. */
SYNTH_API int synth_encode(const float* w, int rows, int cols, uint8_t* q, uint16_t* s)
{
    if (rows <= 0 || cols <= 0 || cols % 64 || !w || !q || !s) return -1;
    int groups = cols / 64;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        for (int g = 0; g < groups; ++g) {
            const float* src = w + (size_t)r * cols + (size_t)g * 64;
            float amax = 0.0f;
            for (int i = 0; i < 64; ++i) { float a = fabsf(src[i]); amax = a > amax ? a : amax; }
            uint16_t s16 = synth_f32_to_f16(amax / 7.0f);
            float sc = synth_f16_to_f32(s16);
            s[(size_t)r * groups + g] = s16;
            uint8_t* dst = q + (size_t)r * (cols / 2) + (size_t)g * 32;
            for (int j = 0; j < 32; ++j) {
                uint32_t nib[2];
                for (int h = 0; h < 2; ++h) {
                    int v = 0;
                    if (sc > 0.0f) {
                        float qq = rintf(src[2 * j + h] / sc);
                        qq = qq < -8.0f ? -8.0f : (qq > 7.0f ? 7.0f : qq);
                        v = (int)qq;
                    }
                    nib[h] = (uint32_t)v & 0x0Fu;
                }
                dst[j] = (uint8_t)(nib[0] | (nib[1] << 4));
            }
        }
    }
    return 0;
}

SYNTH_API int synth_router(uint64_t seed, int layer, int E, int H, float wscale, float* wr)
{
    if (E <= 0 || H <= 0 || !wr) return -1;
    uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_ROUTER, 0, 0);
#pragma omp parallel for schedule(static)
    for (int e = 0; e < E; ++e)
        for (int h = 0; h < H; ++h)
            wr[(size_t)e * H + h] = SYNTH_MUL(wscale, synth_gauss(key, (uint64_t)e * H + h));
    return 0;
}

/* Activations of step `step`: x[t][h] = gauss; bf16 variant rounds to nearest even. */
SYNTH_API int synth_x_f32(uint64_t seed, int step, int T, int H, float* x)
{
    if (T < 0 || H <= 0 || (T && !x)) return -1;
    uint64_t key = synth_key(seed, 0, SYNTH_T_X, (uint32_t)step, 0);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            x[(size_t)t * H + h] = synth_gauss(key, (uint64_t)t * H + h);
    return 0;
}

SYNTH_API int synth_x_bf16(uint64_t seed, int step, int T, int H, uint16_t* x)
{
    if (T < 0 || H <= 0 || (T && !x)) return -1;
    uint64_t key = synth_key(seed, 0, SYNTH_T_X, (uint32_t)step, 0);
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            x[(size_t)t * H + h] = synth_f32_to_bf16(synth_gauss(key, (uint64_t)t * H + h));
    return 0;
}

/*
 * Zipf-skewed router bias: a seeded popularity permutation assigns expert e
 * the rank rank[e] in 1..E; p_r ~ r^-s_exp, and b_e = kappa * ln p_{rank[e]},
 * mean-centred over the experts (so the normalising constant drops out).
 * Writes the bias and, if rank_out != NULL, the ranks.
 */
SYNTH_API int synth_zipf_bias(uint64_t seed, int layer, int E, double kappa, double s_exp,
                              float* bias, int32_t* rank_out)
{
    if (E <= 0 || !bias) return -1;
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    if (!perm) return -2;
    for (int i = 0; i < E; ++i) perm[i] = i;
    uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_PERM, 0, 0);
    /* Fisher-Yates with an unbiased bounded draw (rejection on the top remainder). */
    for (int i = E - 1; i > 0; --i) {
        uint64_t bound = (uint64_t)i + 1u, n = (uint64_t)(E - 1 - i) * 64u, r;
        uint64_t lim = UINT64_MAX - (UINT64_MAX % bound);
        do { r = synth_draw(key, n++); } while (r >= lim);
        int j = (int)(r % bound);
        int32_t tmp = perm[i]; perm[i] = perm[j]; perm[j] = tmp;
    }
    /* perm[r-1] = expert holding popularity rank r */
    double mean = 0.0;
    for (int r = 1; r <= E; ++r) mean += -s_exp * log((double)r);
    mean /= (double)E;
    for (int r = 1; r <= E; ++r) {
        int e = perm[r - 1];
        bias[e] = (float)(kappa * (-s_exp * log((double)r) - mean));
        if (rank_out) rank_out[e] = r;
    }
    free(perm);
    return 0;
}
