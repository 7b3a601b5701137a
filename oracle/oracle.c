/*
 * oracle.c -- plain CPU reference of the int4 expert-FFN MoE layer, fp64.
 *
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU baseline). No blocking, no
 * fusion, no reordering beyond the definitions below; OpenMP only splits
 * independent output elements across threads, each computed in the same order.
 * Shares no code with the CUDA path. See oracle.h for the sources restated.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ---- scalar decoders ------------------------------------------------------ */

/* IEEE binary16: sign, 5-bit exponent (bias 15), 10-bit fraction. */
ORACLE_API double oracle_f16(uint16_t h)
{
    int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0x1F) v = f ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)f, -24);             /* subnormal: f * 2^-24 */
    else v = ldexp((double)(1024 + f), e - 25);             /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16: the top 16 bits of an IEEE binary32. */
ORACLE_API double oracle_bf16(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Element c of a canonical row: byte c/2, low nibble for even c, two's complement. */
ORACLE_API int oracle_code(const uint8_t* row, int c)
{
    int nib = (c & 1) ? (row[c >> 1] >> 4) : (row[c >> 1] & 0x0F);
    return nib >= 8 ? nib - 16 : nib;
}

/* int4 gs64 container ("gs64" groups of 64 along the input dimension, colibri
 * project page, correctness section): W[r][c] = q[r][c] * s[r][c/64]. */
ORACLE_API void oracle_dequant(const uint8_t* q, const uint16_t* s, int rows, int cols, double* w)
{
    int groups = cols / 64;
    for (int r = 0; r < rows; ++r) {
        const uint8_t* row = q + (size_t)r * (cols / 2);
        for (int c = 0; c < cols; ++c)
            w[(size_t)r * cols + c] = (double)oracle_code(row, c) * oracle_f16(s[(size_t)r * groups + c / 64]);
    }
}

static double load_x(const void* x, int xdtype, size_t i)
{
    if (xdtype == ORACLE_BF16) return oracle_bf16(((const uint16_t*)x)[i]);
    return (double)((const float*)x)[i];
}

/* ---- router --------------------------------------------------------------- */

/* Router of the MoE layer (kechuai.cn article, section 一: each layer routes
 * every token to 8 of its 256 experts): l[t][e] = Wr[e] . x[t] + b[e]. */
ORACLE_API void oracle_router_logits(const float* wr, const float* bias, const void* x, int xdtype,
                                     int T, int H, int E, double* logits)
{
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)wr[(size_t)e * H + h] * load_x(x, xdtype, (size_t)t * H + h);
            logits[(size_t)t * E + e] = acc + (bias ? (double)bias[e] : 0.0);
        }
    }
}

typedef struct { double v; int32_t id; } scored;

/* Descending score, equal scores ordered by ascending id. */
static int cmp_scored(const void* a, const void* b)
{
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->id > y->id) - (x->id < y->id);
}

/* Top-K selection by a full sort of all E logits; weights are the softmax over
 * the K selected logits (the router's probabilities renormalised over the
 * selection). A NaN logit is not ordered and is rejected (-1). */
ORACLE_API int oracle_topk(const double* logits, int T, int E, int K, int32_t* ids, double* w)
{
    if (T < 0 || E <= 0 || K <= 0 || K > E) return -1;
    scored* buf = (scored*)malloc(sizeof(scored) * (size_t)E);
    if (!buf) return -1;
    int bad = 0;
    for (int t = 0; t < T && !bad; ++t) {
        for (int e = 0; e < E; ++e) {
            buf[e].v = logits[(size_t)t * E + e];
            buf[e].id = e;
            if (isnan(buf[e].v)) bad = 1;
        }
        qsort(buf, (size_t)E, sizeof(scored), cmp_scored);
        double vmax = buf[0].v, z = 0.0;
        for (int k = 0; k < K; ++k) z += exp(buf[k].v - vmax);
        for (int k = 0; k < K; ++k) {
            ids[(size_t)t * K + k] = buf[k].id;
            if (w) w[(size_t)t * K + k] = exp(buf[k].v - vmax) / z;
        }
    }
    free(buf);
    return bad ? -1 : 0;
}

/* Adaptive expert top-p ("colibri: 1300 lines of C ..." (jsqmd.com), usage
 * section: topp=0.7, adaptive expert top-p, fewer expert reads per token):
 * per token, the experts of the top-K in selection order are kept until
 * their weights (the router probabilities renormalised over the K) sum to at
 * least p; the kept weights are renormalised to sum to 1. */
ORACLE_API int oracle_expert_topp(int T, int K, double p, int32_t* ids, double* w)
{
    int kept_total = 0;
    for (int t = 0; t < T; ++t) {
        int32_t* it = ids + (size_t)t * K;
        double* wt = w + (size_t)t * K;
        int keep = K;
        double cum = 0.0;
        for (int k = 0; k < K; ++k) {
            cum += wt[k];
            if (p < 1.0 && cum >= p) {
                keep = k + 1;
                break;
            }
        }
        for (int k = 0; k < K; ++k) {
            if (k < keep) {
                wt[k] = wt[k] / cum;
            } else {
                wt[k] = 0.0;
                it[k] = -1;
            }
        }
        kept_total += keep;
    }
    return kept_total;
}

ORACLE_API void oracle_weights_full_softmax(const double* logits, int T, int E, int K, const int32_t* ids, double* w)
{
    for (int t = 0; t < T; ++t) {
        const double* l = logits + (size_t)t * E;
        double m = l[0];
        for (int e = 1; e < E; ++e) m = l[e] > m ? l[e] : m;
        double zall = 0.0;
        for (int e = 0; e < E; ++e) zall += exp(l[e] - m);
        double zsel = 0.0;
        for (int k = 0; k < K; ++k) zsel += exp(l[ids[(size_t)t * K + k]] - m) / zall;
        for (int k = 0; k < K; ++k)
            w[(size_t)t * K + k] = (exp(l[ids[(size_t)t * K + k]] - m) / zall) / zsel;
    }
}

/* ---- batch-union ---------------------------------------------------------- */

/* Batch-union (kechuai.cn article, section 二: across the positions of a batch
 * each unique expert is read once): group the T*K routed slots by expert. */
ORACLE_API int oracle_union(const int32_t* ids, int T, int K, int E, int32_t* cnt, int32_t* off,
                            int32_t* unique, int32_t* n_unique, int32_t* pos, int32_t* tok)
{
    for (int i = 0; i < T * K; ++i)
        if (ids[i] < 0 || ids[i] >= E) return -1;
    for (int e = 0; e < E; ++e) cnt[e] = 0;
    for (int i = 0; i < T * K; ++i) cnt[ids[i]] += 1;
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
    int nu = 0;
    for (int e = 0; e < E; ++e)
        if (cnt[e] > 0) unique[nu++] = e;
    *n_unique = nu;
    /* tokens in ascending order: walk t, then k */
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    if (!fill) return -1;
    for (int t = 0; t < T; ++t)
        for (int k = 0; k < K; ++k) {
            int e = ids[(size_t)t * K + k];
            int p = off[e] + fill[e]++;
            pos[(size_t)t * K + k] = p;
            tok[p] = t;
        }
    free(fill);
    return 0;
}

/* ---- expert FFN ----------------------------------------------------------- */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* y_r = sum_c W[r][c] v[c] for one canonical matrix [rows][cols]. */
static void matvec(const uint8_t* q, const uint16_t* s, int rows, int cols, const double* v, double* out)
{
    int groups = cols / 64;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const uint8_t* row = q + (size_t)r * (cols / 2);
        double acc = 0.0;
        for (int c = 0; c < cols; ++c)
            acc += (double)oracle_code(row, c) * oracle_f16(s[(size_t)r * groups + c / 64]) * v[c];
        out[r] = acc;
    }
}

/* An expert is three matrices stored adjacently (kechuai.cn article, section
 * 二); the FFN they form is SwiGLU: h = silu(G x) * (U x), out = D h, with
 * silu(z) = z / (1 + e^-z) and no bias terms. */
ORACLE_API void oracle_expert_ffn(const uint8_t* q, const uint16_t* s, int H, int I, const double* x,
                                  double* out, double* h_out)
{
    size_t mq = (size_t)I * H / 2, ms = (size_t)I * H / 64;
    double* g = (double*)malloc(sizeof(double) * (size_t)I);
    double* u = (double*)malloc(sizeof(double) * (size_t)I);
    double* h = (double*)malloc(sizeof(double) * (size_t)I);
    matvec(q, s, I, H, x, g);
    matvec(q + mq, s + ms, I, H, x, u);
    for (int j = 0; j < I; ++j) h[j] = silu(g[j]) * u[j];
    matvec(q + 2 * mq, s + 2 * ms, H, I, h, out);
    if (h_out) memcpy(h_out, h, sizeof(double) * (size_t)I);
    free(g); free(u); free(h);
}

/* ---- the layer ------------------------------------------------------------ */

static int check_cfg(const oracle_cfg* c)
{
    if (!c || c->hidden <= 0 || c->inter <= 0 || c->hidden % 64 || c->inter % 64) return -1;
    if (c->n_experts <= 0 || c->top_k <= 0 || c->top_k > c->n_experts || c->n_shared < 0) return -1;
    return 0;
}

/* y = shared experts (weight 1: they belong to the always-on dense part,
 * kechuai.cn article section 一) + sum over the K routed experts in routing
 * order, weighted by the renormalised router probabilities. */
static int forward_impl(const oracle_cfg* cfg, const float* wr, const float* bias,
                        const uint8_t* const* eq, const uint16_t* const* es,
                        const void* x, int xdtype, int T, double* y, int32_t* ids_out, double* w_out,
                        int dense)
{
    if (check_cfg(cfg) || T < 0 || !wr || !eq || !es || (T && (!x || !y))) return -1;
    if (xdtype != ORACLE_F32 && xdtype != ORACLE_BF16) return -1;
    int H = cfg->hidden, I = cfg->inter, E = cfg->n_experts, K = cfg->top_k;
    if (T == 0) return 0;
    double* logits = (double*)malloc(sizeof(double) * (size_t)T * E);
    int32_t* ids = (int32_t*)malloc(sizeof(int32_t) * (size_t)T * K);
    double* w = (double*)malloc(sizeof(double) * (size_t)T * K);
    double* xt = (double*)malloc(sizeof(double) * (size_t)H);
    double* o = (double*)malloc(sizeof(double) * (size_t)H);
    int rc = 0;
    if (!logits || !ids || !w || !xt || !o) { rc = -1; goto done; }
    oracle_router_logits(wr, bias, x, xdtype, T, H, E, logits);
    if (oracle_topk(logits, T, E, K, ids, w)) { rc = -1; goto done; }
    if (cfg->expert_top_p > 0.0 && cfg->expert_top_p < 1.0) oracle_expert_topp(T, K, cfg->expert_top_p, ids, w);
    for (int i = 0; i < T * K; ++i)
        if (ids[i] >= 0 && (!eq[ids[i]] || !es[ids[i]])) { rc = -2; goto done; }
    for (int t = 0; t < T; ++t) {
        double* yt = y + (size_t)t * H;
        for (int h = 0; h < H; ++h) { xt[h] = load_x(x, xdtype, (size_t)t * H + h); yt[h] = 0.0; }
        for (int j = 0; j < cfg->n_shared; ++j) {
            oracle_expert_ffn(eq[E + j], es[E + j], H, I, xt, o, NULL);
            for (int h = 0; h < H; ++h) yt[h] += o[h];
        }
        if (!dense) {
            for (int k = 0; k < K; ++k) {
                int e = ids[(size_t)t * K + k];
                if (e < 0) continue; /* dropped by expert top-p */
                oracle_expert_ffn(eq[e], es[e], H, I, xt, o, NULL);
                for (int h = 0; h < H; ++h) yt[h] += w[(size_t)t * K + k] * o[h];
            }
        } else {
            /* every expert, gate weight zero unless selected (then its weight) */
            for (int e = 0; e < E; ++e) {
                double ge = 0.0;
                for (int k = 0; k < K; ++k)
                    if (ids[(size_t)t * K + k] == e) ge = w[(size_t)t * K + k];
                if (!eq[e] || !es[e]) { rc = -2; goto done; }
                oracle_expert_ffn(eq[e], es[e], H, I, xt, o, NULL);
                for (int h = 0; h < H; ++h) yt[h] += ge * o[h];
            }
        }
    }
    if (ids_out) memcpy(ids_out, ids, sizeof(int32_t) * (size_t)T * K);
    if (w_out) memcpy(w_out, w, sizeof(double) * (size_t)T * K);
done:
    free(logits); free(ids); free(w); free(xt); free(o);
    return rc;
}

ORACLE_API int oracle_moe_forward(const oracle_cfg* cfg, const float* wr, const float* bias,
                                  const uint8_t* const* eq, const uint16_t* const* es,
                                  const void* x, int xdtype, int T, double* y, int32_t* ids, double* w)
{
    return forward_impl(cfg, wr, bias, eq, es, x, xdtype, T, y, ids, w, 0);
}

ORACLE_API int oracle_moe_forward_dense(const oracle_cfg* cfg, const float* wr, const float* bias,
                                        const uint8_t* const* eq, const uint16_t* const* es,
                                        const void* x, int xdtype, int T, double* y)
{
    return forward_impl(cfg, wr, bias, eq, es, x, xdtype, T, y, NULL, NULL, 1);
}

/* ---- residual stack ------------------------------------------------------- */

/* RMSNorm with unit gain. The pages give no normalisation for a stack of MoE
 * layers; a pre-norm residual is the plainest one that keeps activations finite. */
ORACLE_API void oracle_rmsnorm(const double* x, int T, int H, double eps, double* out)
{
    for (int t = 0; t < T; ++t) {
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += x[(size_t)t * H + h] * x[(size_t)t * H + h];
        double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int h = 0; h < H; ++h) out[(size_t)t * H + h] = x[(size_t)t * H + h] * r;
    }
}

ORACLE_API int oracle_stack_step(const oracle_cfg* cfg, const float* wr, const float* bias,
                                 const uint8_t* const* eq, const uint16_t* const* es,
                                 float* x, int T, double eps, int32_t* ids)
{
    if (check_cfg(cfg) || T < 0 || (T && !x)) return -1;
    if (T == 0) return 0;
    int H = cfg->hidden;
    size_t n = (size_t)T * H;
    double* xd = (double*)malloc(sizeof(double) * n);
    double* nd = (double*)malloc(sizeof(double) * n);
    float* nf = (float*)malloc(sizeof(float) * n);
    double* y = (double*)malloc(sizeof(double) * n);
    int rc = -1;
    if (xd && nd && nf && y) {
        for (size_t i = 0; i < n; ++i) xd[i] = (double)x[i];
        oracle_rmsnorm(xd, T, H, eps, nd);
        for (size_t i = 0; i < n; ++i) nf[i] = (float)nd[i];
        rc = oracle_moe_forward(cfg, wr, bias, eq, es, nf, ORACLE_F32, T, y, ids, NULL);
        if (rc == 0)
            for (size_t i = 0; i < n; ++i) x[i] = (float)(xd[i] + y[i]);
    }
    free(xd); free(nd); free(nf); free(y);
    return rc;
}
