/*
 * coli_moe.h -- C ABI of the int4 expert-FFN MoE layer for one NVIDIA B200.
 *
 * The layer is the sparse MoE block of the Colibri engine pages:
 *   "Colibri: 2400 lines of pure C ..." (kechuai.cn/articles/colibri),
 *     section 一: every layer routes each token to 8 of its 256 experts; the
 *     shared expert belongs to the always-on dense part; an int4 expert is
 *     about 19 MB; section 二: an expert's three matrices are stored
 *     adjacently and a batch reads each unique expert once (batch-union);
 *   "colibri" project page (gh.puless.com/p/colibri.html), section on
 *     correctness: the int4 container uses groups of 64 (gs64).
 * Readings where the pages are silent: router scores are the logits
 * Wr x + b; the top-k is taken in descending logit order, equal logits going
 * to the lower expert id; routing weights are the softmax over the k selected
 * logits; each expert is a SwiGLU FFN  D (silu(G x) * (U x)); shared experts
 * have weight 1; y = sum(shared) + sum_k w_k E_k(x).
 *
 * Conventions
 *  - Every call returns a coli_status. Argument errors return COLI_EINVAL
 *    before any work is enqueued and change nothing. CUDA failures return
 *    COLI_ECUDA; coli_last_error() gives the message (thread-local).
 *    The library never prints, exits or aborts.
 *  - A `coli_stream` is a cudaStream_t passed as void* (NULL: legacy default
 *    stream). Route and forward are asynchronous and stream-ordered; their
 *    tensor arguments are DEVICE pointers on the layer's device.
 *  - A layer owns its weights and a workspace sized for cfg.max_tokens. The
 *    workspace is single-stream: calls on one layer must not overlap.
 *  - Dimensions: hidden % 128 == 0, inter % 64 == 0, group_size == 64,
 *    1 <= top_k <= n_experts <= 1024, n_shared >= 0, max_tokens >= 1.
 */
#ifndef COLI_MOE_H
#define COLI_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_EINVAL = 1,       /* bad argument (null, size, alignment, dtype)      */
    COLI_ENOMEM = 2,       /* device or host allocation failed                  */
    COLI_ECUDA = 3,        /* a CUDA call or kernel launch failed               */
    COLI_EUNSUPPORTED = 4  /* valid request this build does not implement       */
} coli_status;

typedef enum { COLI_F32 = 0, COLI_BF16 = 1 } coli_dtype;

typedef void* coli_stream; /* cudaStream_t */

typedef struct {
    int hidden;      /* H: model width (input of gate/up, output of down)           */
    int inter;       /* I: expert intermediate width                               */
    int n_experts;   /* E: routed experts (256 in the pages' model)                */
    int top_k;       /* K: experts per token (8 in the pages' model)               */
    int n_shared;    /* always-on shared experts, weight 1 each                    */
    int group_size;  /* must be 64: one fp16 scale per 64 inputs of a row          */
    int max_tokens;  /* largest n_tokens a route/forward call may pass             */
} coli_moe_config;

typedef struct coli_moe_layer coli_moe_layer; /* opaque */

/*
 * Create a layer on `device` from canonical weights.
 *
 * router_w    [E][H] fp32, row-major.
 * router_bias [E] fp32, or NULL for zero bias. The bias enters the logits, so
 *             it moves both the selection and the weights.
 * expert_q    canonical int4 weights of the E routed experts, expert after
 *             expert; one expert is  gate [I][H/2] | up [I][H/2] | down [H][I/2]
 *             bytes (3*H*I/2 per expert). Byte j of a row holds elements 2j
 *             (low nibble) and 2j+1 (high nibble) as two's complement codes.
 * expert_scales  fp16 bit patterns, expert after expert:
 *             gate [I][H/64] | up [I][H/64] | down [H][I/64] (3*H*I/64 per
 *             expert); element c of row r is code(r, c) * scale(r, c/64).
 * shared_q / shared_scales  the n_shared shared experts, same layout (NULL
 *             when n_shared == 0).
 * Every input pointer may be host or device memory (detected per pointer) and
 * is only read during the call; the caller keeps ownership. expert_q and
 * shared_q may be NULL (with their scales NULL) to create a layer whose
 * experts are loaded afterwards with coli_moe_layer_set_experts.
 * The call is synchronous. On failure *out is NULL and nothing leaks.
 */
coli_status coli_moe_layer_create(const coli_moe_config* cfg, const float* router_w, const float* router_bias,
                                  const uint8_t* expert_q, const uint16_t* expert_scales,
                                  const uint8_t* shared_q, const uint16_t* shared_scales,
                                  int device, coli_moe_layer** out);

/*
 * (Re)load `count` experts starting at expert id `first` (routed ids
 * 0..E-1, shared ids E..E+n_shared-1) from canonical buffers holding `count`
 * consecutive experts (layout as in coli_moe_layer_create; host or device).
 * Synchronous.
 */
coli_status coli_moe_layer_set_experts(coli_moe_layer* layer, int first, int count,
                                       const uint8_t* q, const uint16_t* scales);

void coli_moe_layer_destroy(coli_moe_layer* layer);

/*
 * Expert cache: a layer whose routed experts do not all stay in HBM.
 * The Colibri pages keep the hot experts in fast memory and fetch the others
 * on demand ("Colibri: 2400 lines of pure C ..." (kechuai.cn), section 二: a
 * per-layer cache with least-recently-used eviction, a hot set learned from
 * routing counts that stays pinned, and the next layer's router run one
 * layer ahead to prefetch; project page (gh.puless.com/p/colibri.html),
 * placement tiers). Here HBM is the cache and page-locked host memory the
 * store behind it.
 *
 * Arguments as coli_moe_layer_create, plus resident_slots R with
 * min(n_experts, max_tokens * top_k) <= R <= n_experts; expert_q and
 * expert_scales must not be NULL. HBM holds R routed experts and the shared
 * experts; every routed expert is also kept, in the device layout, in
 * page-locked host memory (n_experts * stride bytes, stride about
 * coli_moe_expert_bytes rounded up to 256). Experts 0..R-1 start resident.
 *
 * coli_moe_forward on a cached layer routes the batch, reads the ids back
 * (the call waits for them, so it cannot be captured in a CUDA graph), makes
 * every routed expert the batch needs resident, then runs the resident
 * layer's kernels through the slot table with that routing. A missing expert
 * takes a free slot, else the slot whose expert was used least recently among
 * those neither pinned nor needed by the batch; it arrives by one
 * cudaMemcpyAsync of its gate/up and down matrices (adjacent) on the
 * forward's stream. The output equals a resident layer's for the same
 * routing, bit for bit. coli_moe_stack_forward over cached layers also runs
 * each next layer's router on the current layer's input and prefetches the
 * experts it picks on that layer's own copy stream while the current layer's
 * kernels run (see coli_moe_cache_set_lookahead).
 * coli_moe_layer_set_experts on a cached layer updates the host copy (and the
 * HBM copy when resident).
 */
coli_status coli_moe_layer_create_cached(const coli_moe_config* cfg, const float* router_w, const float* router_bias,
                                         const uint8_t* expert_q, const uint16_t* expert_scales,
                                         const uint8_t* shared_q, const uint16_t* shared_scales,
                                         int resident_slots, int device, coli_moe_layer** out);

/*
 * Expert parallelism (an MoE layer sharded by expert over `world` GPUs, one
 * process per GPU): rank r holds the routed experts
 * [E*r/world, E*(r+1)/world) (coli_moe_ep_range) and, on rank 0 only, the
 * shared experts. Arguments as coli_moe_layer_create (expert_q and
 * expert_scales hold all E experts in the canonical layout; only this rank's
 * are read; shared_q is read on rank 0 only), plus rank and world
 * (1 <= world <= n_experts).
 *
 * The router is replicated: every rank computes the full top-K of every token.
 * A forward then writes this rank's PARTIAL output,
 *   y_r[t] = [r == 0] * sum_j shared_j(x_t) + sum over the token's slots k
 *            whose expert this rank holds of w[t][k] * E_ids[t][k](x_t),
 * with the same kernels as a whole layer (the plan lists only this rank's
 * experts; the other slots are empty: coli_moe_get_plan reports them as id
 * -1 and position -1). The caller sums y_r over the ranks (an all-reduce, for
 * example NCCL over NVLink); the sum is the layer's output up to the order of
 * the fp32 additions. A bf16 layer's partial outputs are bf16.
 * coli_moe_route on such a layer returns the full routing.
 */
coli_status coli_moe_layer_create_ep(const coli_moe_config* cfg, const float* router_w, const float* router_bias,
                                     const uint8_t* expert_q, const uint16_t* expert_scales,
                                     const uint8_t* shared_q, const uint16_t* shared_scales,
                                     int rank, int world, int device, coli_moe_layer** out);

/* The routed experts [*first, *end) that rank `rank` of `world` holds. */
coli_status coli_moe_ep_range(int n_experts, int rank, int world, int* first, int* end);

typedef struct {
    int64_t hits;           /* experts a batch needed that were resident                */
    int64_t misses;         /* experts a batch needed that were copied in before it     */
    int64_t bytes_h2d;      /* expert bytes copied from host memory (misses + prefetch)  */
    int64_t prefetched;     /* experts copied ahead of need (lookahead, prefetch, pin)   */
    int64_t prefetch_used;  /* of those, the ones a batch needed before their eviction   */
    int64_t predicted;      /* needed experts that the lookahead prediction named        */
    int64_t predicted_of;   /* needed experts of the forwards that had a prediction      */
    int32_t resident_slots; /* R                                                         */
    int32_t n_pinned;       /* experts pinned by coli_moe_cache_pin                      */
} coli_cache_stats;

/*
 * Counters of a cached layer since creation or the last reset (reset != 0
 * clears them after reading; the usage counts are kept). usage: NULL or
 * [n_experts] int64, the number of batches that routed to each expert since
 * creation: the learned hot set (save it across sessions and pass its top
 * entries to coli_moe_cache_pin). Waits for the layer's copies in flight.
 * COLI_EINVAL on a layer that is not cached.
 */
coli_status coli_moe_cache_stats(coli_moe_layer* layer, coli_cache_stats* stats, int64_t* usage, int reset);

/*
 * Pins the n experts ids[0..n) (host int32; n == 0 unpins all): they become
 * resident now and are never evicted. At most
 * R - min(n_experts, max_tokens * top_k) experts may be pinned, so that any
 * batch still fits. Synchronous.
 */
coli_status coli_moe_cache_pin(coli_moe_layer* layer, const int32_t* ids, int n);

/*
 * Copies the distinct experts among ids[0..n) (host int32) into HBM ahead of
 * need, on the layer's copy stream, evicting by the same rule as a forward
 * (as many as fit). Returns at once; the next forward waits for the copies.
 */
coli_status coli_moe_cache_prefetch(coli_moe_layer* layer, const int32_t* ids, int n);

/* The cache slot of each routed expert (host int32 [n_experts]; -1: not in
 * HBM), as placed by the calls made so far (copies may still be in flight). */
coli_status coli_moe_cache_slots(const coli_moe_layer* layer, int32_t* slots);

/* Whether this cached layer accepts the previous stack layer's lookahead
 * prediction (1, the default) or not (0). */
coli_status coli_moe_cache_set_lookahead(coli_moe_layer* layer, int enable);

/* Copy of the layer's configuration. */
coli_status coli_moe_layer_config(const coli_moe_layer* layer, coli_moe_config* cfg);

/*
 * Router only: ids[t][k] (int32) and weights[t][k] (fp32, summing to 1 per
 * token) for x [n_tokens][H] (fp32 or bf16 bits). 0 <= n_tokens <= max_tokens.
 * Below 64 tokens the logits are accumulated in fp64 from the exact products
 * of fp32 inputs. From 64 tokens, where the layer allows it, the certified
 * router (coli_moe_router_fallbacks) computes them exactly up to a rigorous
 * per-logit bound and falls back to fp64 for every token the bound does not
 * settle. Equal logits go to the lower id; the ids and their order can differ
 * from those of the exact logits only for logits closer than fp64 rounding.
 */
coli_status coli_moe_route(coli_moe_layer* layer, const void* x, coli_dtype dtype, int n_tokens,
                           int32_t* ids, float* weights, coli_stream stream);

/*
 * The layer: y [n_tokens][H] = MoE(x), y of the same dtype as x. x and y must
 * not overlap. Paths (see coli_moe_set_fused and coli_moe_set_tensor_cores):
 *  - up to 64 tokens (and at most 512 routed slots, n_tokens * top_k): one
 *    persistent kernel runs the whole layer on integer tensor-core MMAs. Each
 *    64-input group of a token (or of a SwiGLU output row) is encoded as a
 *    15-bit signed integer times a power of two chosen from the group's
 *    largest magnitude (relative step 2^-15 of that magnitude), split into two
 *    signed 8-bit parts; the int4 weights enter as their codes, each group's
 *    sum is exact in 32-bit integers, and the group scales, the SwiGLU and the
 *    combine are fp32. The output is deterministic.
 *  - larger bf16 batches: the tcgen05 tensor-core grouped GEMMs (fp16
 *    operands: tokens scaled by powers of two and converted exactly, weights
 *    rounded once to fp16, fp32 accumulation; the combine adds with fp32
 *    atomics, so the summation order, and the last bits of y, may vary
 *    between runs). The tensor-core path needs an sm_100 device,
 *    hidden % 256 == 0, inter % 128 == 0 and weight scales of magnitude
 *    <= 4096; otherwise bf16 also runs the CUDA-core kernels.
 *  - larger fp32 batches: the CUDA-core kernels (fp32 arithmetic).
 * Sparse-expert forward as the Colibrì pages describe it (top-8 of 256 routed
 * experts plus the always-on shared expert, each distinct expert's int4
 * weights read once per batch).
 */
coli_status coli_moe_forward(coli_moe_layer* layer, const void* x, void* y, coli_dtype dtype, int n_tokens,
                             coli_stream stream);

/*
 * Residual stack over fp32 activations, in place:
 *   x <- x + MoE_l(RMSNorm(x)) for l = 0..n_layers-1,
 * RMSNorm with unit gain: x / sqrt(mean(x^2) + eps). All layers must share
 * H and live on one device; n_tokens <= every layer's max_tokens.
 */
coli_status coli_moe_stack_forward(coli_moe_layer* const* layers, int n_layers, float* x, int n_tokens,
                                   float eps, coli_stream stream);

/*
 * Statistics of the last forward on this layer (synchronises its stream):
 * number of distinct routed experts, bytes of expert and router weights the
 * plan streams ((unique + n_shared) * expert bytes + router bytes), and, if
 * per_expert_counts != NULL, the routed-slot count of each of the E experts.
 */
coli_status coli_moe_get_stats(coli_moe_layer* layer, int* n_unique, int64_t* bytes_streamed,
                               int32_t* per_expert_counts);

/*
 * Number of kernels of this library that route, forward and stack calls on
 * this layer have enqueued since it was created (load-time kernels and the
 * driver memset that clears the tensor-core path's fp32 output are not
 * counted). Host-side counter: no synchronisation. n must not be NULL
 * (COLI_EINVAL).
 */
coli_status coli_moe_get_launch_count(const coli_moe_layer* layer, int64_t* n);

/*
 * The batch-union plan of the last forward (synchronises; host outputs, any
 * of them NULL to skip):
 *   ids [T][K], weights [T][K]      routing
 *   counts [E], offsets [E+1]       slots per expert and their exclusive scan
 *   unique [E], *n_unique           distinct experts, ascending
 *   pos [T][K]                      position of slot (t,k) in the permuted list
 *   tok [T*K]                       token of each permuted position
 * T is the n_tokens of that forward.
 */
coli_status coli_moe_get_plan(coli_moe_layer* layer, int32_t* ids, float* weights, int32_t* counts,
                              int32_t* offsets, int32_t* unique, int32_t* n_unique, int32_t* pos, int32_t* tok);

/*
 * The certified router of token batches (batches of 64 tokens and more, on a
 * device and with shapes that allow it: H a multiple of 16 in [128, 65536],
 * E <= 256): router rows and tokens as four signed 8-bit digit planes under
 * power-of-two row scales, every logit from one exact int8 tensor-core GEMM
 * with a rigorous bound of its representation error, and the top-K, its
 * order and its weights taken from those logits when the bounds prove them
 * ("Colibri: 2400 lines of pure C ..." (kechuai.cn), section 一, defines the
 * router and its top-K). A token whose selection the bounds do not settle (a
 * near tie at or above the K-th place, a weight bound above 5e-7, with
 * expert top-p a running sum within the bound of p, or a non-finite input)
 * gets all of its logits and its top-K in fp64 instead.
 * *certified: 1 when this layer routes such batches with it, else 0.
 * *n: tokens of the last batch it routed that took the fp64 fallback (0 when
 * it is not in use). Synchronises with the device: call after the routing
 * finished (coli_moe_sync, or a synchronisation of the stream it ran on).
 * Either output may be NULL.
 */
coli_status coli_moe_router_fallbacks(coli_moe_layer* layer, int32_t* certified, int32_t* n);

/*
 * Per-stage device timing of forward calls, for profiling. While enabled,
 * every forward records CUDA events between its kernels on its own stream
 * (no host synchronisation; a ring of event sets is recycled, folding each
 * finished forward into running totals). coli_moe_get_profile waits for the
 * profiled forwards to finish and writes, per stage, the total device ms over
 * all forwards since profiling was enabled, and their number. Enabling again
 * resets the totals. On the tensor-core path the plan stage also covers the
 * operand rows, the tile list and the clear of the fp32 output, so the
 * gate/up and down stages each time one grouped-GEMM kernel alone. The cache
 * stage (cached layers) runs from the routed ids' read-back to the kernels:
 * the next layer's lookahead routing, the copies of missing experts and the
 * slot table upload, plus the host's wait for the ids.
 */
enum { COLI_STAGE_ROUTER = 0, COLI_STAGE_TOPK, COLI_STAGE_PLAN, COLI_STAGE_GATEUP, COLI_STAGE_DOWN,
       COLI_STAGE_COMBINE, COLI_STAGE_FUSED, COLI_STAGE_CACHE, COLI_N_STAGES };
coli_status coli_moe_set_profiling(coli_moe_layer* layer, int enable);
coli_status coli_moe_get_profile(coli_moe_layer* layer, double* stage_ms_total, int64_t* n_forwards);
const char* coli_moe_stage_name(int stage);

/*
 * Waits for the layer's last forward. Returns COLI_ECUDA if the persistent
 * decode kernel gave up on a bounded wait (its inputs are then invalid); the
 * layer is reset and stays usable. get_stats and get_plan do the same check.
 */
coli_status coli_moe_sync(coli_moe_layer* layer);

/*
 * Selects the path for small batches: 1 (default) runs the whole layer for up
 * to 64 tokens in one persistent kernel on integer MMAs (router, top-k, plan,
 * experts, combine); 0 runs the separate kernels. Routing is identical;
 * outputs agree within rounding. Returns COLI_EUNSUPPORTED when the shapes do
 * not fit the kernel's shared memory, COLI_EINVAL for another value.
 */
coli_status coli_moe_set_fused(coli_moe_layer* layer, int enable);

/*
 * Path for batches of more than 4 tokens: mode 0 the CUDA-core kernels for
 * both dtypes; 1 (default) the tcgen05 tensor-core kernels for bf16; 2 the
 * tensor cores for fp32 as well, each fp32 token entering as an fp16 hi + lo
 * pair (about 22 bits; weights and the SwiGLU output h are fp16, so a layer's
 * relative error is a few 1e-4 against the fp32 kernels' 1e-6). Returns
 * COLI_EUNSUPPORTED for modes 1 and 2 when the device, the shapes or the
 * weight scales rule the tensor-core path out.
 */
coli_status coli_moe_set_tensor_cores(coli_moe_layer* layer, int mode);

/*
 * Adaptive expert top-p, opt-in ("colibri: 1300 lines of C ..." (jsqmd.com),
 * usage section: topp=0.7, adaptive expert top-p, 30-40% fewer expert reads).
 * It changes the routing: with 0 < p < 1, after the top-K of a token (slots
 * in descending logit order, weights w_k renormalised over the K) the slots
 * are kept while the running sum of w in slot order (fp64) has not reached p,
 * the slot that reaches it included; the kept weights are divided by that
 * sum. A dropped slot reports slot 0's id with weight 0 (route, plan and
 * forward alike): the batch-union reads no expert for it and the combine
 * adds exactly 0. p = 1 (the default) is the plain top-K. Applies to
 * coli_moe_route, coli_moe_forward and the stack on this layer (not to
 * coli_moe_route_noalloc). p outside (0, 1] returns COLI_EINVAL.
 */
coli_status coli_moe_set_expert_top_p(coli_moe_layer* layer, double p);

/*
 * Item timeline of the persistent decode kernel, for profiling. `buffer` is a
 * caller-owned DEVICE buffer of 8 * (16 + 8 * capacity) bytes, zeroed by the
 * caller; int64 [0] counts records (it may exceed capacity: later records are
 * dropped); [1..8] global-timer stamps of the plan path: [1] the last router
 * item seen done, [2] after its counter update, [3] plan published, [4] top-k
 * started, [5] top-k done, [6] counts and scans done, [7] positions written,
 * [8] before the release of the plan flag; [9] the earliest CTA start (atomic
 * minimum: the caller sets it to INT64_MAX), [10] the last CTA's exit, [11]
 * the latest end of an output block's combine.
 * Record r at int64 16 + 8r: {cta << 40 | kind << 32 | expert << 16 | tile,
 * begin ns, end ns, ns waited for the item's first weight stage, tokens of the
 * item, total ns consumer 0 waited for weight stages, weight loop start ns,
 * weight loop end ns (0 for items without weights)}; kind 1
 * router rows, 2 gate/up tile, 3 down tile, 4 token quantisation; times from
 * the GPU global timer. NULL disables tracing.
 * In a library built with COLI_TC_TRACE=1 (a profiling build; the default
 * build records nothing there), the tensor-core path writes, with
 * c = (capacity - 256) / 16 when positive,
 * the timeline of CTA 0 of its gate/up launch at int64 0 and of its down
 * launch at int64 8c + 128: per 64-input block b < c, 8 SM clock stamps at
 * 8b (transform warp has the block, its A stage is free, its stores issued,
 * MMA thread has the block, has the A stage, issued; producer has the stage,
 * issued the copies), then per work item i < 64 two stamps at 8c + 2i
 * (epilogue start, end).
 */
coli_status coli_moe_set_trace(coli_moe_layer* layer, void* buffer, int capacity);

/*
 * Weight-streaming geometry of the persistent decode kernel: each SM keeps up
 * to `stages` bulk copies of at most `blocks_per_stage` x 4352 bytes in flight
 * (defaults 3 and 16; what fits in shared memory beside the token operands:
 * two copies of 16 blocks up to 32 tokens, three of 8 blocks above).
 * stages in [2, 24], blocks_per_stage even in [2, 16]. A tuning knob: results
 * do not change.
 */
coli_status coli_moe_set_ring(coli_moe_layer* layer, int stages, int blocks_per_stage);

/*
 * Routing that allocates nothing (no counterpart in the paper: an
 * integration aid). For callers that cannot call cudaMalloc where they
 * route: code running while a stream is captured into a CUDA graph, code
 * that lives on a fixed memory budget from another framework's pool, or
 * paths that must not wait on the driver's allocator. It needs no layer:
 * router_w [n_experts][hidden] fp32 and router_bias [n_experts] fp32 (or
 * NULL) are DEVICE pointers the caller owns, as are x [n_tokens][hidden]
 * (fp32 or bf16 bits), ids [n_tokens][top_k] and weights [n_tokens][top_k];
 * the results equal coli_moe_route's for the same inputs (the logits are
 * summed in the same order).
 * Its only scratch, the fp64 logits, is a fixed 504 KiB array in device
 * memory that every GPU loading this library holds until the process exits:
 * n_tokens <= COLI_NOALLOC_MAX_TOKENS and n_experts <= COLI_NOALLOC_MAX_EXPERTS,
 * larger requests return COLI_EINVAL. All calls on a device share that array,
 * so calls that overlap on the GPU (different streams without ordering) race
 * and give wrong results; order them on one stream. The first call on each
 * device looks the array's device address up (cudaGetSymbolAddress, with that
 * device current): make that first call before any stream capture. The
 * address is looked up again when the device's context has changed (after a
 * cudaDeviceReset); make the first call after a reset outside a capture too.
 * Asynchronous on `stream`; argument errors return before any work.
 */
#define COLI_NOALLOC_MAX_TOKENS 63
#define COLI_NOALLOC_MAX_EXPERTS 1024
coli_status coli_moe_route_noalloc(const float* router_w, const float* router_bias, int n_experts, int hidden,
                                   int top_k, const void* x, coli_dtype dtype, int n_tokens, int32_t* ids,
                                   float* weights, coli_stream stream);

/*
 * Testing aid for the bounded waits of the kernels that wait on barriers or
 * flags (the integer-MMA persistent kernel, the certified router's GEMM and the
 * tensor-core grouped GEMMs): every wait of their launches on this layer gives
 * up after wait_ns nanoseconds (0: the default, 1 s), and with enable != 0 one
 * gate/up item of each persistent launch waits on a flag that nothing sets, and
 * one MMA warp of each GEMM launch on a barrier that nothing completes, so the
 * launches give up: their CTAs drain their copies and exit, and coli_moe_sync
 * then returns COLI_ECUDA (naming the site of the first wait that gave up) and
 * resets the layer, which stays usable. No GPU fault or hang is involved.
 */
coli_status coli_moe_debug_wait_test(coli_moe_layer* layer, int enable, int64_t wait_ns);

/*
 * Testing aid for the out-of-memory paths: from now on, the nth device or
 * page-locked host allocation this library makes for a layer (create,
 * set_experts) fails as if that memory were exhausted; 0 disables. The failing call returns
 * COLI_ENOMEM, frees what it had allocated, and create leaves *out NULL.
 * Process-wide; nth < 0 returns COLI_EINVAL.
 */
coli_status coli_moe_debug_fail_alloc(int nth);

/*
 * Measurement aid: enqueues one kernel of n_blocks blocks (one per SM is the
 * intent; launch as many as the device has SMs) in which block b writes
 * {SM id, SM clock counter, global timer in ns} as int64 at buffer[3 b ..].
 * Two stamps around a timed region give each SM's mean clock rate there:
 * (clock difference) / (timer difference) for blocks on the same SM.
 * buffer: DEVICE memory of 3 * n_blocks int64; 1 <= n_blocks <= 65535.
 */
coli_status coli_clock_stamp(long long* buffer, int n_blocks, coli_stream stream);

/* Bytes of one expert in the int4 gs64 container (nibbles + fp16 scales). */
int64_t coli_moe_expert_bytes(int hidden, int inter);

const char* coli_status_string(coli_status status);
/* Detail of the last failure on the calling thread ("" if none). */
const char* coli_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* COLI_MOE_H */
