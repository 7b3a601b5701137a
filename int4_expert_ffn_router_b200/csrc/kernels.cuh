// kernels.cuh -- launchers of the CUDA path (defined in router.cu, ffn_core.cu,
// repack.cu, combine.cu).
#pragma once

#include <string>

#include "common.cuh"

namespace coli {

// router.cu
// From this batch size on (with a partial-sum scratch) the router uses the
// blocked GEMM form, which sums each logit in another order.
constexpr int kRouterGemmMinTok = 64;
// part: optional scratch of part_cap doubles for split-input partial sums
// (batches of kRouterGemmMinTok tokens and more use the blocked GEMM form).
cudaError_t launch_router_logits(const float* wr, const float* bias, const void* x, coli_dtype dt, int T, int H, int E,
                                 double* logits, cudaStream_t st, double* part = nullptr, size_t part_cap = 0);
// The router of token batches on the integer tensor cores with a certified
// selection (router_certified.cu): Wr and x as four signed 8-bit digit planes
// under power-of-two row scales, every logit from one exact int8 GEMM with a
// rigorous bound of its representation error, the top-K, its order and its
// weights taken from those logits where the bounds prove them, and the fp64
// logits and top-K for the other tokens. Five kernels.
struct RouterCert {
    uint8_t* maps = nullptr;       // host: 6 CUtensorMap (router planes; batch planes for 5 tile heights), 64-byte aligned
    uint8_t* wd8 = nullptr;        // [4][E][H] router digit planes
    int* wscale = nullptr;         // [E] row scale exponents r_e
    double* wb = nullptr;          // [E][3] ||Wr_e - wh_e||, ||wh_e||, rounding-bound factor
    uint8_t* xd8 = nullptr;        // [4][Tm][H] batch digit planes
    int* xscale = nullptr;         // [Tm] token scale exponents s_t
    double* xb = nullptr;          // [Tm][3] ||x_t||, ||x_t - xh_t||, ||xh_t||
    int* fail = nullptr;           // [1 + Tm]: count, then the tokens sent to the fp64 fallback
    int Tm = 0, H = 0, E = 0, n_sm = 148;
};
bool router_certified_supported(int H, int E);
size_t router_certified_smem_bytes();
// Digit planes and bound factors of the router rows, the tensor maps (once).
cudaError_t router_certified_prepare(RouterCert& rc, const float* wr, cudaStream_t st);
// err: timeout site of the GEMM's bounded waits (control block); wait_ns: their
// bound (0: 1 s); wait_test: testing aid, the GEMM's MMA warp first waits on a
// barrier that nothing completes, so the launch gives up and reports a timeout.
cudaError_t launch_router_certified(const RouterCert& rc, const float* wr, const float* bias, const void* x,
                                    coli_dtype dt, int T, int K, double topp, int e_lo, int e_hi, double* logits,
                                    int32_t* ids, float* w, int* err, int64_t wait_ns, int wait_test,
                                    cudaStream_t st);
// Kernels launch_router_logits enqueues for these arguments (0, 1 or 2).
int router_kernel_count(int T, int H, int E, const double* part, size_t part_cap);
// topp in (0, 1): adaptive expert top-p after the top-K (topk.cuh, topk_weights); else plain top-K.
// Selected experts outside [e_lo, e_hi) (e_hi < 0: E) are written as empty slots (id -1).
cudaError_t launch_topk(const double* logits, int T, int E, int K, int32_t* ids, float* w, cudaStream_t st,
                        double topp = 1.0, int e_lo = 0, int e_hi = -1);
size_t plan_smem_bytes(int E);
cudaError_t launch_plan(const int32_t* ids, int T, int K, int E, int S, const Plan& p, cudaStream_t st);

// repack.cu: canonical matrix [R][C] (nibbles + fp16 scales, device memory)
// into the device layout. `interleave_gu`: src0 = gate [I][H], src1 = up
// [I][H], written as one [2I][H] matrix interleaved by 8 rows.
cudaError_t launch_repack(const uint8_t* q0, const uint16_t* s0, const uint8_t* q1, const uint16_t* s1, int R, int C,
                          bool interleave_gu, uint8_t* dst, cudaStream_t st);

// ffn_core.cu: CUDA-core int4 expert matrices over the active experts.
// Gate/up + SwiGLU: h[pos][I] (fp32) for every active (expert, token).
cudaError_t launch_gateup_core(const uint8_t* weights, const Dims& d, const void* x, coli_dtype dt, int T,
                               const Plan& p, float* h, int max_active, int n_sm, cudaStream_t st);
// Down: o[pos][H] (fp32) for every active (expert, token).
cudaError_t launch_down_core(const uint8_t* weights, const Dims& d, const float* h, int T, const Plan& p, float* o,
                             int max_active, int n_sm, cudaStream_t st);

// Persistent decode kernel ring defaults: bulk copies in flight per SM and
// 4352-byte blocks per copy (coli_moe_set_ring).
constexpr int kDefaultStages = 3;
constexpr int kDefaultStageBlocks = 16;

// decode_i8.cu: the whole layer for 1..kI8MaxTok tokens (at most kI8MaxSlots
// routed slots) in one persistent launch of n_sm CTAs, on integer MMAs.
constexpr int kI8MaxTok = 64;
constexpr int kI8MaxSlots = 512;
struct I8Launch {
    const uint8_t* weights;
    Dims d;
    const float* wr;
    const float* bias;
    const void* x;
    coli_dtype dt;
    int T;
    void* y;
    const float* residual;
    Plan p;
    double* logits;
    const int32_t* given_ids;  // [T][K] ids routed before the launch (then no router items run), or NULL
    const float* given_w;      // [T][K] their weights
    double topp;               // adaptive expert top-p of the in-kernel routing (>= 1 or 0: plain top-K)
    int ep_lo, ep_hi;          // routed experts of this rank (expert parallelism): others become empty slots
    uint8_t* xq;   // [T][H/64][128] token parts (written by the kernel)
    uint8_t* xm;   // [T][H/64][16]
    uint8_t* hq;   // [slots][I/64][128] SwiGLU output parts
    uint8_t* hm;   // [slots][I/64][16]
    float* o;      // [slots][H]
    int* ctl;      // control block of i8_ctl_ints_for(d, T) ints, zero at launch (left zero but a timeout code)
    int n_sm;
    size_t smem_limit;
    long long* trace;
    int trace_cap;
    int max_stages, max_sb;
    int64_t wait_ns;  // bound of every wait (<= 0: 1 s)
    int wait_test;    // testing aid: one gate/up item waits on a flag that nothing sets
};
cudaError_t launch_decode_i8(const I8Launch& l, cudaStream_t st);
bool decode_i8_supported(const Dims& d, int T, size_t smem_limit);
int i8_ctl_ints_for(const Dims& d, int T);

// prefill_tc.cu: the expert FFNs of a bf16 token batch on the tensor cores.
// meta: [0] max over gate/up row pairs of L1(gate row) * L1(up row) (float
// bits), [1] max |scale| (float bits); folded in per expert by launch_l1_bound
// from the canonical container (device memory).
cudaError_t launch_l1_bound(const uint8_t* q, const uint16_t* s, int H, int I, unsigned* meta, cudaStream_t st);
// xs[p] = fp16(x[t] * 2^e_t) for every position p of token t (its K routed
// positions and one per shared expert), tscale[t] = {2^-e_t, 2^f_t, 2^-f_t, 0}.
// fp32 x: two rows per position (2p hi, 2p + 1 lo).
cudaError_t launch_prefill_prep(const void* x, coli_dtype dt, int T, int H, int K, int S, const int32_t* pos,
                                const float* meta, __half* xs, float4* tscale, cudaStream_t st);
// Per-position epilogue factors and the tile list.
cudaError_t launch_prefill_plan(const Plan& p, int T, int K, int S, int max_tok, const float4* tscale, float4* slot,
                                int4* tiles, int* n_tiles, cudaStream_t st);
// phase 0: h16 = fp16(2^f silu(G x) (U x)); phase 1: y32 += (w / 2^f) D h16.
// token_maps: host copies of two 2D tensor maps (make_token_map; boxes of
// kTcMaxTok and 32 rows) over xs (phase 0) or h16 (phase 1).
// pairs (phase 0): the operand holds hi and lo rows per position (fp32 input).
// wait_ns: bound of the kernel's waits (0: 1 s); wait_test: testing aid, one MMA warp first
// waits on a barrier that nothing completes, so the launch gives up and reports a timeout.
cudaError_t launch_prefill_gemm(int phase, bool pairs, const uint8_t* weights, const Dims& d, const void* token_maps,
                                const Plan& p, const float4* slot, const int4* tiles, const int* n_tiles, __half* h16,
                                float* y32, int* err, int n_sm, long long* trace, int trace_cap, int64_t wait_ns,
                                int wait_test, cudaStream_t st);
// Encodes a 2D fp16 tensor map (128 bytes, written to `map`) over
// [rows][cols] at `base`: box 64 x box_rows, 128-byte swizzle.
cudaError_t make_token_map(void* map, const void* base, int rows, int cols, int box_rows);
constexpr int kTensorMapBytes = 128;
// y = y32 (+ residual), stored as fp32 or bf16.
cudaError_t launch_prefill_out(const float* y32, const float* residual, int T, int H, void* y, coli_dtype dt,
                               cudaStream_t st);
size_t prefill_tc_smem_bytes();
int prefill_tc_max_tiles(const Dims& d, int T);

// layer.cu: record the message coli_last_error() returns on this thread.
void set_last_error(const std::string& what);

// combine.cu
// y[t] = residual[t] (optional) + sum_j o[TK + j*T + t] + sum_k w[t][k] o[pos[t][k]]
cudaError_t launch_combine(const float* o, const Plan& p, int T, int H, int K, int S, const float* residual, void* y,
                           coli_dtype ydt, cudaStream_t st);
// out[t] = x[t] / sqrt(mean(x[t]^2) + eps), fp64 statistics, fp32 output
cudaError_t launch_rmsnorm(const float* x, int T, int H, float eps, float* out, cudaStream_t st);

}  // namespace coli
