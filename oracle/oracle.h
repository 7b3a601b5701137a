/*
 * oracle.h -- plain CPU reference of the int4 expert-FFN MoE layer.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's CPU
 * baseline use this library; the product path never links, loads or calls it.
 * It shares no code with the CUDA path (the two only read the same seeded
 * input bytes).
 *
 * Everything accumulates in fp64. The method it restates is the sparse MoE
 * layer of the Colibri engine pages:
 *   - "Colibri: 2400 lines of pure C ..." (kechuai.cn/articles/colibri),
 *     section 一 (background): 256 routed experts per layer, 8 routed per token,
 *     the shared expert is part of the always-resident dense part, ~19 MB per
 *     int4 expert; section 二 (mechanism): the three matrices of an expert are
 *     stored adjacently, and a batch reads each unique expert once (batch-union).
 *   - "colibri" project page (gh.puless.com/p/colibri.html), section
 *     "aggressive optimisation, conservative correctness": the int4 container
 *     uses groups of 64 (gs64); sparse selection is validated by forcing full
 *     selection and comparing with the dense computation.
 * Readings the pages leave open (router softmax renormalised over the top-k,
 * ties to the lower expert id, SwiGLU expert, shared-expert weight 1, RMSNorm
 * pre-norm for a residual stack) are stated at each function.
 *
 * Canonical expert buffer (per expert, the three matrices adjacent):
 *   q: gate [I][H/2] | up [I][H/2] | down [H][I/2]   bytes; byte j of a row holds
 *      elements 2j (low nibble) and 2j+1 (high nibble), two's complement
 *   s: gate [I][H/64] | up [I][H/64] | down [H][I/64] fp16 bits, one per group of
 *      64 consecutive elements along the row (the input dimension)
 */
#ifndef COLI_ORACLE_H
#define COLI_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int hidden;     /* H */
    int inter;      /* I */
    int n_experts;  /* E, routed */
    int top_k;      /* K */
    int n_shared;   /* shared experts, weight 1 each */
    double expert_top_p; /* adaptive expert top-p (oracle_expert_topp); 0 or >= 1: off */
} oracle_cfg;

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* fp16 / bf16 bit patterns to double (exact). */
double oracle_f16(uint16_t h);
double oracle_bf16(uint16_t b);
/* Signed value of element `c` of a canonical row (two's complement nibble). */
int oracle_code(const uint8_t* row, int c);
/* W[r][c] = code(r, c) * scale(r, c / 64), exact in fp64. */
void oracle_dequant(const uint8_t* q, const uint16_t* s, int rows, int cols, double* w);

/* l[t][e] = sum_h Wr[e][h] x[t][h] + b[e]   (b may be NULL: zero bias) */
void oracle_router_logits(const float* wr, const float* bias, const void* x, int xdtype,
                          int T, int H, int E, double* logits);
/* K largest logits per token, descending, ties to the lower id; weights are the
 * softmax over the selected logits. Returns 0, or -1 on bad sizes. */
int oracle_topk(const double* logits, int T, int E, int K, int32_t* ids, double* w);
/* Adaptive expert top-p on a top-K result (ids and weights [T][K] in
 * selection order, weights summing to 1 per token): keep the shortest prefix
 * whose weights sum (in order, fp64) to at least p, renormalise the kept
 * weights by that sum, and mark the dropped slots id -1, weight 0. At least
 * one expert is kept; p >= 1 keeps all K. Returns the number of slots kept. */
int oracle_expert_topp(int T, int K, double p, int32_t* ids, double* w);
/* Second form of the weights: softmax over all E logits, renormalised over the
 * selected ids (self-check of oracle_topk's weights). */
void oracle_weights_full_softmax(const double* logits, int T, int E, int K, const int32_t* ids, double* w);

/* Batch-union plan of ids [T][K]:
 *   cnt[e] = number of slots routed to e; off = exclusive scan of cnt (E+1);
 *   unique = experts with cnt > 0, ascending (n_unique of them);
 *   pos[t*K+k] = off[e] + rank of t among e's tokens (tokens ascending);
 *   tok[pos]   = t (the permuted token list).  Returns 0 or -1 on bad ids. */
int oracle_union(const int32_t* ids, int T, int K, int E, int32_t* cnt, int32_t* off,
                 int32_t* unique, int32_t* n_unique, int32_t* pos, int32_t* tok);

/* One expert on one token: g = G x, u = U x, h = silu(g) * u, out = D h.
 * h_out (I doubles) may be NULL. */
void oracle_expert_ffn(const uint8_t* q, const uint16_t* s, int H, int I, const double* x,
                       double* out, double* h_out);

/* The layer: y[t] = sum_j shared_j(x_t) + sum_k w[t][k] * E_ids[t][k](x_t),
 * the routed sum taken in routing order; with cfg->expert_top_p in (0, 1) the
 * routing is reduced by oracle_expert_topp first (dropped slots: id -1). eq/es hold E + n_shared expert pointers
 * (routed 0..E-1, then shared); a routed entry may be NULL if never selected.
 * ids/w may be NULL. Returns 0, -1 on bad arguments, -2 if a selected expert is NULL. */
int oracle_moe_forward(const oracle_cfg* cfg, const float* wr, const float* bias,
                       const uint8_t* const* eq, const uint16_t* const* es,
                       const void* x, int xdtype, int T, double* y, int32_t* ids, double* w);
/* Brute force: every routed expert evaluated, gate weight 0 off the selection. */
int oracle_moe_forward_dense(const oracle_cfg* cfg, const float* wr, const float* bias,
                             const uint8_t* const* eq, const uint16_t* const* es,
                             const void* x, int xdtype, int T, double* y);

/* RMSNorm with unit gain: out = x / sqrt(mean(x^2) + eps). */
void oracle_rmsnorm(const double* x, int T, int H, double eps, double* out);
/* One residual stack step on an fp32 stream: x <- fp32(x + MoE(rmsnorm(x))),
 * with the normalised input rounded to fp32 (the layer input is fp32). */
int oracle_stack_step(const oracle_cfg* cfg, const float* wr, const float* bias,
                      const uint8_t* const* eq, const uint16_t* const* es,
                      float* x, int T, double eps, int32_t* ids);

#ifdef __cplusplus
}
#endif
#endif
