// decode_i8.cu -- the whole MoE layer for up to 64 tokens in one persistent
// kernel: token quantisation, router, top-k, batch-union plan, int4 gate/up +
// SwiGLU, down, and the weighted combine with the shared expert.
//
// Decode streams each active expert's ~20 MB once ("Colibri: 2400 lines of
// pure C ...", kechuai.cn, section 二: one read per unique expert per batch,
// the three matrices stored adjacently), so the kernel must keep HBM busy and
// keep every per-weight instruction count far below what HBM speed allows
// (about 41 weights per SM clock at 6.5 TB/s). One CTA per SM, three roles:
//  * a producer thread takes work tickets and streams each item's 128-row
//    weight tile into a shared-memory ring with bulk asynchronous copies; at
//    one or two tokens it also copies the next item's token operands into a
//    second buffer while the current item streams;
//  * eight consumer warps (one 16-row sub-tile each) multiply on the tensor
//    cores from registers with integer MMAs (mma.m16n8k32, u8 x s8 -> s32):
//    the weights enter as their offset-binary codes (one logic op per four
//    weights), the tokens as two signed 8-bit parts of a 15-bit fixed-point
//    value per 64-input group (block floating point: one power-of-two scale
//    per group and token), and each group's sum is exact in 32-bit integers
//    before the fp16 group scale and the token scale are applied in fp32;
//  * a signaler warp publishes completions (release atomics) and combines
//    each 128-row block of y when its last down tile lands.
// A work item is one 128-row weight tile of one expert for up to 8 of its
// tokens (the MMA's 8 B columns hold 4 tokens x 2 parts; two column chunks).
// Tickets come in dependency order: token quantisation, router rows, shared
// gate/up, then (once the plan is published) routed gate/up, shared down,
// routed down. An item only waits for items with smaller tickets, which
// running CTAs already hold; every wait is bounded in time and reports a
// timeout through the control block instead of hanging.
#include <string>

#include "common.cuh"
#include "kernels.cuh"
#include "topk.cuh"

namespace coli {
namespace {

constexpr int kSub = 8;                      // 16-row sub-tiles of a 128-row weight tile
// One consumer warp per sub-tile: ten warps per CTA leave 158 registers per
// thread, where two warps per sub-tile (on alternate blocks) left 96 and spilled
// in the weight loop (measured 2.5% slower at batch 1, 5% at batch 8).
constexpr int kWS = 1;                       // consumer warps per sub-tile
constexpr int kCW = kSub * kWS;              // consumer warps
constexpr int kCT = kCW * 32;                // consumer threads
constexpr int kProducerWarp = kCW;
constexpr int kSignalWarp = kCW + 1;
constexpr int kFT = (kCW + 2) * 32;          // all threads
constexpr int kMaxSB = 8;                    // 4352-byte blocks per ring stage (at most)
constexpr int kQ = 2;                        // item queue slots (lookahead of one item)
constexpr int kSQ = 4;                       // completion records in flight to the signaler
constexpr int kRouterExperts = 2;            // experts per router item (kCW / 2 warps each)
static_assert(kWS == 1 || kWS == 2, "one or two consumer warps per sub-tile");
constexpr int kChunkTok = 4;                 // tokens per 8-column MMA chunk (hi and lo parts)
constexpr int kMetaRow = 16;                 // bytes of one group's data {2^-e, -8 sum(hi), -8 sum(lo), 0}
// In shared memory each token slot's group data is followed by one unused
// 16-byte entry, so the four tokens of an MMA chunk fall in different banks.
__host__ __device__ constexpr size_t meta_slot_bytes(int G) { return (size_t)(G + 1) * kMetaRow; }

enum { IT_END = 0, IT_PREP = 1, IT_ROUTER = 2, IT_GU = 3, IT_DOWN = 4 };

// Control block (ints, zero between launches).
// Each word that many CTAs poll or update gets its own 128-byte line, so
// pollers of one do not slow the atomics on another.
enum {
    kCI_Ticket = 0, kCI_Router = 32, kCI_Plan = 64, kCI_Exit = 96, kCI_Error = kCtlError, kCI_Prep = 160,
    kCI_Never = 192,  // never set: the testing aid of coli_moe_debug_wait_test waits on it
    kCI_Counters = 224
};

struct Item {
    int kind;
    int ex;      // expert (routed id or E + shared index); prep: token
    int rt;      // 128-row tile
    int chunk;   // chunk id: shared chunks first, then routed chunks
    int pos;     // first position of the chunk
    int cnt;     // tokens of the chunk (<= 8)
    int tok0;    // shared chunk: its first token; routed: -1 (tokens from the plan)
    int ready;   // down: gate/up of the chunk already complete when published
    int staged;  // two B buffers: the producer issued the B operands' copies into this slot's buffer
};

struct I8Args {
    const uint8_t* weights;
    Dims d;
    const float* wr;
    const float* bias;
    const void* x;
    void* y;
    const float* residual;
    int T;
    Plan p;
    double* logits;
    const int32_t* given_ids;  // [T][K] routing computed before the launch (expert cache), or NULL
    const float* given_w;      // [T][K] its weights
    double topp;               // adaptive expert top-p of the in-kernel routing (>= 1: plain top-K)
    int ep_lo, ep_hi;          // routed experts of this rank; the others become empty slots (id -1)
    uint8_t* xq;   // [T][H/64][128]  token limbs
    uint8_t* xm;   // [T][H/64][16]   token group meta
    uint8_t* hq;   // [slots][I/64][128]
    uint8_t* hm;   // [slots][I/64][16]
    float* o;      // [slots][H] fp32 expert outputs
    int* ctl;
    int ntc;       // tokens per item (4 or 8)
    int cps;       // chunks per shared expert: ceil(T / ntc)
    int ncmax;     // bound on routed chunks
    int nstages;   // ring stages
    int sb;        // 4352-byte blocks per stage
    int nbuf;      // B buffers: 2 (one per item-queue slot) when two items' operands fit, else 1
    int nbt;       // positions one B buffer holds (ntc with one buffer)
    int64_t wait_ns;   // bound of every wait
    int wait_test;     // nonzero: the first gate/up tile waits on a flag nothing sets (testing aid)
    long long* trace;  // item timeline (NULL: off)
    int trace_cap;
};

// Control block layout after the fixed words.
__host__ __device__ inline int i8_ctl_gu(int) { return kCI_Counters; }                 // [chunks] gate/up tiles done
__host__ __device__ inline int i8_ctl_dn(int nchunks) { return kCI_Counters + nchunks; }  // [H/128] down tiles done
__host__ __device__ inline int i8_ctl_entries(int nchunks, int H) { return (kCI_Counters + nchunks + H / 128 + 1) & ~1; }
__host__ __device__ inline int i8_ctl_ints(int nchunks, int H, int ncmax) { return i8_ctl_entries(nchunks, H) + 2 * ncmax; }

struct I8Smem {
    uint64_t full[kMaxStages], empty[kMaxStages], qfull[kQ], qempty[kQ], dfull[kSQ], dempty[kSQ], bfull;
    uint64_t bslot_full[kQ];   // two B buffers: one phase per item of the queue slot
    int bslot_pending[kQ];     // copies into the buffer issued and not yet seen complete
    uint32_t bslot_parity[kQ]; // parity of that phase
    Item items[kQ];
    Item cur[2];
    Item done[kSQ];
    int abort_flag;
    int last;
    uint32_t bphase;        // B stagings completed (parity of bfull)
    int bpending;           // a B staging was issued and not yet seen complete
    int aborted;            // snapshot of abort_flag taken by consumer 0 before a barrier
    int staged_kind;        // IT_GU / IT_DOWN / -1: what the B area holds
    int plan_chunks;        // routed chunks of the plan this CTA built
    int staged_n, staged_key;
    int staged_tok[8];
    int wsum[kCW], wflag[kCW];
    float hmaxw[kSub][8];   // gate/up epilogue: per sub-tile, max |h| of each token of the item
    int hsum[kSub][8][2];   // per sub-tile, sums of the hi and lo parts of each token
    alignas(16) float accx[kSub][32][4];  // partial sums of the second warp of each sub-tile (read as float4)
    unsigned long long first_wait_ns, total_wait_ns;
    unsigned long long t_loop0, t_loop1;  // trace: the item's weight loop started / ended
};

// ------------------------------------------------------------- small helpers
__device__ __forceinline__ int atom_add_acq_rel(int* p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ void red_add_release(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Orders this thread's earlier (acquired) view of global memory before its
// later bulk asynchronous copies read it.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void set_error(I8Args& a, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    atomicCAS(&a.ctl[kCI_Error], 0, code);
}

// True when another CTA has given up (its timeout code is in the control
// block): this CTA stops too instead of waiting out its own bounds.
__device__ __forceinline__ bool others_gave_up(I8Args& a, volatile int* abort_flag) {
    if (*reinterpret_cast<volatile int*>(&a.ctl[kCI_Error]) == 0) return false;
    *abort_flag = 1;
    return true;
}

// Bounded wait on an mbarrier phase; gives up when the CTA aborts, when
// another CTA gave up, or after a.wait_ns.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, I8Args& a,
                                         int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((n & 63) == 0 && others_gave_up(a, abort_flag)) return false;
        if (globaltimer_ns() - t0 > (uint64_t)a.wait_ns) {
            set_error(a, abort_flag, code);
            return false;
        }
    }
}

// Bounded wait until *p >= target (acquire), polling every ~64 ns: the
// waits on the plan and on the prepared tokens are on the critical path, so
// the poll interval stays short (a longer backoff measurably lengthened the
// batch-1 step).
__device__ __forceinline__ bool wait_geq(const int* p, int target, volatile int* abort_flag, I8Args& a, int code) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        __nanosleep(64);
        if (ld_acquire(p) >= target) return true;
        if (*abort_flag) return false;
        if ((n & 7) == 0 && others_gave_up(a, abort_flag)) return false;
        if (globaltimer_ns() - t0 > (uint64_t)a.wait_ns) {
            set_error(a, abort_flag, code);
            return false;
        }
    }
}

__device__ __forceinline__ unsigned long long* entries_of(I8Args& a, int nchunks) {
    return reinterpret_cast<unsigned long long*>(a.ctl + i8_ctl_entries(nchunks, a.d.H));
}

// Byte offset, within one 64-byte part of a group, of input k (0..63): the
// order in which a lane's 16 bytes feed mma.m16n8k32 as B fragments, matching
// the weight layout's lane slots (lane 4 gi + ti of a sub-tile holds, in word
// s, the inputs 16 s + {2 ti, 2 ti + 8, 2 ti + 1, 2 ti + 9} of rows gi, gi+8).
__device__ __forceinline__ int limb_offset(int k) {
    const int s = k >> 4, r = k & 15;
    const int hiq = r >> 3, rr = r & 7;         // inputs 8..15 of the 16-input step
    const int t = rr >> 1, odd = rr & 1;        // k = 16 s + 2 t + odd (+ 8 hiq)
    const int b = odd * 2 + hiq;                // byte within the 4-byte word
    return t * 16 + 4 * s + b;
}

// 2^k as a float, k in [-126, 127] (exponent bits written directly).
__device__ __forceinline__ float pow2f(int k) { return __uint_as_float((uint32_t)(127 + k) << 23); }

// Exponent e of the block-floating-point encoding of a group whose largest
// magnitude is m: m 2^e in [2^14, 32639], so that rint(v 2^e) = 256 hi + lo
// with hi, lo in [-128, 127]. 0 for m = 0 (and for non-finite m).
__device__ __forceinline__ int group_exponent(float m) {
    const uint32_t b = __float_as_uint(m);
    const int be = (int)((b >> 23) & 0xFF);
    if (m <= 0.0f || be == 0xFF) return 0;
    int e;
    if (be == 0) {  // subnormal: m < 2^-126, the largest shift keeps every product finite
        e = 126;
    } else {
        e = 14 - (be - 127);  // m 2^e in [2^14, 2^15)
        e = e > 126 ? 126 : (e < -126 ? -126 : e);
        // m 2^e = 2^14 (1 + f): above 32639 when the 23-bit fraction exceeds 0x7EFE00
        if (e == 14 - (be - 127) && (b & 0x7FFFFFu) > 0x7EFE00u) e -= 1;
    }
    return e;
}

// Block-floating-point encoding of one 64-input group of one token (or
// position), one warp, lane l holding inputs 2l and 2l+1 (v0, v1): scale 2^e
// with max |v| 2^e in [2^14, 32639], integer x = rint(v 2^e) split as
// x = 256 hi + lo with hi, lo in [-128, 127]. Writes the two 64-byte parts
// (hi, then lo) at `dst` and {2^-e, -8 sum(hi), -8 sum(lo), 0} at `meta`.
__device__ __forceinline__ void encode_group(float v0, float v1, uint8_t* dst, uint8_t* meta, int lane) {
    float m = fmaxf(fabsf(v0), fabsf(v1));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = group_exponent(m);
    const float f = pow2f(e);
    int hi[2], lo[2];
    const float v[2] = {v0, v1};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int xi = __float2int_rn(v[i] * f);
        hi[i] = (xi + 128) >> 8;
        lo[i] = xi - 256 * hi[i];
        const int k = 2 * lane + i;
        dst[limb_offset(k)] = (uint8_t)(int8_t)hi[i];
        dst[64 + limb_offset(k)] = (uint8_t)(int8_t)lo[i];
    }
    int sh = hi[0] + hi[1], sl = lo[0] + lo[1];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sh += __shfl_xor_sync(0xffffffffu, sh, o);
        sl += __shfl_xor_sync(0xffffffffu, sl, o);
    }
    if (lane == 0) *reinterpret_cast<int4*>(meta) = make_int4(__float_as_int(pow2f(-e)), -8 * sh, -8 * sl, 0);
}

// u8 x s8 -> s32 MMA, 16 x 8 x 32, accumulating in place.
__device__ __forceinline__ void mma_u8s8(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Number of routed chunks and the shared-chunk count of a launch.
struct Phases {
    int P, R, SC, RTgu, RTd, Ggu, Gd, t_sgu, t_dyn, nch;
};
__device__ __forceinline__ Phases phases_of(const I8Args& a) {
    Phases f;
    const Dims& d = a.d;
    f.P = a.T;
    f.R = a.given_ids ? 0 : (d.E + kRouterExperts - 1) / kRouterExperts;
    f.SC = d.S * a.cps;
    f.RTgu = 2 * d.I / kTileRows;
    f.RTd = d.H / kTileRows;
    f.Ggu = d.H / kGroup;
    f.Gd = d.I / kGroup;
    f.t_sgu = f.P + f.R;
    f.t_dyn = f.t_sgu + f.SC * f.RTgu;
    f.nch = f.SC + a.ncmax;
    return f;
}

// The shared chunk sc: tokens ntc (sc % cps) .. of shared expert sc / cps.
__device__ __forceinline__ Item shared_chunk(const I8Args& a, int kind, int sc, int rt) {
    const int j = sc / a.cps, c = sc % a.cps;
    const int tok0 = c * a.ntc;
    const int cnt = min(a.ntc, a.T - tok0);
    return Item{kind, a.d.E + j, rt, sc, a.T * a.d.K + j * a.T + tok0, cnt, tok0, 0};
}

// Token i of a gate/up item: shared chunks hold consecutive tokens; routed
// chunks read theirs from the published plan (with one token, token 0).
__device__ __forceinline__ int item_token(const I8Args& a, const Item& it, int i) {
    return it.tok0 >= 0 ? it.tok0 + i : a.T == 1 ? 0 : __ldcg(a.p.tok + it.pos + i);
}

// B buffers in the B area, each the operands of a.nbt positions (limbs, then
// group data): one buffer of ntc positions, or two (one per item-queue slot)
// of the largest chunk a launch can form.
__device__ __forceinline__ uint8_t* buf_limbs(const I8Args& a, uint8_t* barea, int k) {
    const int G = (a.d.H > a.d.I ? a.d.H : a.d.I) / kGroup;
    return barea + (size_t)k * a.nbt * ((size_t)G * 128 + meta_slot_bytes(G));
}
__device__ __forceinline__ uint8_t* buf_meta(const I8Args& a, uint8_t* barea, int k) {
    const int G = (a.d.H > a.d.I ? a.d.H : a.d.I) / kGroup;
    return buf_limbs(a, barea, k) + (size_t)a.nbt * G * 128;
}

// Two B buffers: the copies of weight item it's B operands (token limbs and
// group data for gate/up, h rows for down) into the buffer of queue slot k,
// completing the slot's phase of the given parity. The caller (the producer,
// or consumer 0 when the inputs were not ready at publication) has acquired
// the completion of whatever wrote them.
__device__ void stage_slot(I8Args& a, I8Smem& S, const Item& it, int k, uint32_t parity, uint8_t* barea) {
    const Phases f = phases_of(a);
    const bool gu = it.kind == IT_GU;
    const int G = gu ? f.Ggu : f.Gd, nt = it.cnt;
    if (nt > a.nbt) {  // cannot happen when the host sized the buffers; never write past one
        set_error(a, &S.abort_flag, kCtlErrBufferOverflow);
        return;
    }
    uint8_t* lb = buf_limbs(a, barea, k);
    uint8_t* mb = buf_meta(a, barea, k);
    uint64_t* bar = &S.bslot_full[k];
    fence_proxy_async_global();
    const uint32_t lbytes = (uint32_t)G * 128, mbytes = (uint32_t)G * kMetaRow;
    S.bslot_parity[k] = parity;
    S.bslot_pending[k] = 1;
    mbar_arrive_expect_tx(bar, (uint32_t)nt * (lbytes + mbytes));
    if (gu) {
        for (int i = 0; i < nt; ++i) {
            const int tok = item_token(a, it, i);
            bulk_g2s(lb + (size_t)i * lbytes, a.xq + (size_t)tok * lbytes, lbytes, bar);
            bulk_g2s(mb + (size_t)i * meta_slot_bytes(G), a.xm + (size_t)tok * mbytes, mbytes, bar);
        }
    } else {
        bulk_g2s(lb, a.hq + (size_t)it.pos * lbytes, nt * lbytes, bar);
        for (int i = 0; i < nt; ++i)
            bulk_g2s(mb + (size_t)i * meta_slot_bytes(G), a.hm + (size_t)(it.pos + i) * mbytes, mbytes, bar);
    }
}

// ------------------------------------------------------------------ producer
__device__ void i8_producer(I8Args& a, I8Smem& S, uint8_t* ring) {
    const Dims& d = a.d;
    const Phases f = phases_of(a);
    volatile int* abort_flag = &S.abort_flag;
    const unsigned long long* entries = entries_of(a, f.nch);
    uint32_t q = 0, gs = 0, slot_s = 0, phase_s = 0;
    bool first_ticket = true;
    bool prep_seen = false;  // every token's quantisation is complete (acquired)
    uint8_t* barea = ring + (size_t)a.nstages * a.sb * kBlockBytes;
    const uint64_t wpolicy = l2_policy_evict_first();
    int nc = -1;  // routed chunks, once the plan is published
    while (true) {
        Item it{IT_END, 0, 0, 0, 0, 0, -1, 0};
        if (!*abort_flag) {
            // the first ticket of CTA b is b (no contended atomic at start-up); later ones
            // come from the shared counter, after the gridDim.x static ones
            const int t = first_ticket ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(&a.ctl[kCI_Ticket], 1);
            first_ticket = false;
            if (t < f.P) {
                it = Item{IT_PREP, t, 0, 0, 0, 1, t, 0};
            } else if (t < f.t_sgu) {
                it.kind = IT_ROUTER;
                it.ex = (t - f.P) * kRouterExperts;
            } else if (t < f.t_dyn) {
                it = shared_chunk(a, IT_GU, (t - f.t_sgu) / f.RTgu, (t - f.t_sgu) % f.RTgu);
            } else {
                if (nc < 0 && wait_geq(&a.ctl[kCI_Plan], 1, abort_flag, a, 2)) nc = ld_acquire(&a.ctl[kCI_Plan]) - 1;
                int dd = t - f.t_dyn;
                if (nc < 0) {
                    it.kind = IT_END;  // aborted
                } else if (dd < nc * f.RTgu || (dd >= nc * f.RTgu + f.SC * f.RTd &&
                                                dd < nc * (f.RTgu + f.RTd) + f.SC * f.RTd)) {
                    const bool gu = dd < nc * f.RTgu;
                    const int RT = gu ? f.RTgu : f.RTd;
                    const int r = gu ? dd : dd - nc * f.RTgu - f.SC * f.RTd;
                    const int c = r / RT;
                    const unsigned long long v = __ldcg(entries + c);
                    it = Item{gu ? IT_GU : IT_DOWN, (int)(v & 0xFFFF), r % RT, f.SC + c, (int)((v >> 16) & 0xFFFFF),
                              (int)((v >> 36) & 0xF), -1, 0};
                } else if (dd >= nc * f.RTgu && dd < nc * f.RTgu + f.SC * f.RTd) {
                    dd -= nc * f.RTgu;
                    it = shared_chunk(a, IT_DOWN, dd / f.RTd, dd % f.RTd);
                }
            }
            if (it.kind == IT_DOWN) it.ready = ld_acquire(&a.ctl[i8_ctl_gu(f.nch) + it.chunk]) >= f.RTgu;
        }
        const uint32_t slot = q % kQ;
        if (q >= kQ && !wait_bar(&S.qempty[slot], ((q / kQ) - 1) & 1, abort_flag, a, 3)) it.kind = IT_END;
        if (a.nbuf == 2) {
            // the slot's buffer is free (the consumers are done with the slot's previous item):
            // stage a weight item's B operands now when their inputs are complete, so that the
            // consumers find them landed; otherwise consumer 0 stages them. Every other item
            // completes the slot's phase with a plain arrival (one phase per item), except
            // after an abort, when the slot's last phase may still wait for copies in flight
            // and nothing but the exit drain waits on it.
            const bool w = it.kind == IT_GU || it.kind == IT_DOWN;
            bool ready = false;
            if (w && !*abort_flag) {
                if (it.kind == IT_GU) {
                    if (!prep_seen) prep_seen = ld_acquire(&a.ctl[kCI_Prep]) >= f.P;
                    // the testing aid's item keeps the consumers' staging path, where it waits
                    ready = prep_seen && !(a.wait_test && it.chunk == 0 && it.rt == 0);
                } else {
                    ready = it.ready != 0;
                }
            }
            if (ready) {
                stage_slot(a, S, it, (int)slot, (q / kQ) & 1, barea);
                it.staged = 1;
            } else if (!w && !*abort_flag) {
                mbar_arrive(&S.bslot_full[slot]);
            }
        }
        S.items[slot] = it;
        mbar_arrive(&S.qfull[slot]);
        ++q;
        if (it.kind == IT_END) break;
        // Router and quantisation items read global memory with plain loads, which would
        // queue behind this SM's in-flight weight copies: stream nothing until they are done.
        if ((it.kind == IT_ROUTER || it.kind == IT_PREP) &&
            !wait_bar(&S.qempty[slot], ((q - 1) / kQ) & 1, abort_flag, a, 12))
            continue;
        if (it.kind == IT_GU || it.kind == IT_DOWN) {
            const bool gu = it.kind == IT_GU;
            const int G = gu ? f.Ggu : f.Gd;
            const uint8_t* tile = a.weights + expert_offset(d, it.ex) + (gu ? 0 : d.gu_bytes) +
                                  (size_t)it.rt * G * kBlockBytes;
            const uint32_t stage_bytes = (uint32_t)a.sb * kBlockBytes;
            for (int b0 = 0; b0 < G; b0 += a.sb) {
                const int nb = min(a.sb, G - b0);
                // slot_s = gs % nstages, phase_s = (gs / nstages) & 1
                if (gs >= (uint32_t)a.nstages && !wait_bar(&S.empty[slot_s], phase_s ^ 1, abort_flag, a, 4)) break;
                mbar_arrive_expect_tx(&S.full[slot_s], nb * kBlockBytes);
                // weights are read once: they leave L2 first, ahead of the token limbs, h rows and
                // expert outputs that other CTAs read again
                bulk_g2s_policy(ring + (size_t)slot_s * stage_bytes, tile + (size_t)b0 * kBlockBytes, nb * kBlockBytes,
                                &S.full[slot_s], wpolicy);
                ++gs;
                if (++slot_s == (uint32_t)a.nstages) { slot_s = 0; phase_s ^= 1; }
            }
        }
    }
    // let the copies in flight land before the CTA exits (bounded)
    const uint32_t ns = a.nstages;
    for (uint32_t k = (gs > ns ? gs - ns : 0); k < gs; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&S.full[k % ns], (k / ns) & 1) && globaltimer_ns() - t0 < (uint64_t)a.wait_ns) {
        }
    }
}

// ------------------------------------------------------------------ signaler
// y rows of output block rt: residual + shared experts + routed experts in
// routing order (fixed order, as the separate combine kernel).
template <typename XT>
__device__ void signal_combine(I8Args& a, int rt, int lane) {
    const Dims& d = a.d;
    const int T = a.T, K = d.K, TK = T * d.K;
    constexpr int kJ = kTileRows / 32;  // rows per lane: rt * 128 + 32 j + lane
    for (int t = 0; t < T; ++t) {
        float acc[kJ];
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const int r = rt * kTileRows + j * 32 + lane;
            acc[j] = a.residual ? a.residual[(size_t)t * d.H + r] : 0.0f;
        }
        for (int s = 0; s < d.S; ++s) {
            const float* os = a.o + (size_t)(TK + s * T + t) * d.H + rt * kTileRows + lane;
            float v[kJ];
#pragma unroll
            for (int j = 0; j < kJ; ++j) v[j] = __ldcg(os + 32 * j);
#pragma unroll
            for (int j = 0; j < kJ; ++j) acc[j] += v[j];
        }
        // routed slots 32 at a time: lane k holds the position and weight of slot k0 + k;
        // the slots' rows are read together, then added in routing order
        for (int k0 = 0; k0 < K; k0 += 32) {
            const int nk = min(32, K - k0);
            const int q_l = lane < nk ? __ldcg(a.p.pos + t * K + k0 + lane) : 0;
            const float w_l = lane < nk ? __ldcg(a.p.w + t * K + k0 + lane) : 0.0f;
            for (int c0 = 0; c0 < nk; c0 += 8) {
                float v[8][kJ];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int qq = __shfl_sync(0xffffffffu, q_l, (c0 + c) & 31);
                    const float* orow = a.o + (size_t)max(qq, 0) * d.H + rt * kTileRows + lane;
                    // an empty slot (qq < 0: expert of another rank) reads nothing and adds 0
#pragma unroll
                    for (int j = 0; j < kJ; ++j) v[c][j] = (c0 + c < nk && qq >= 0) ? __ldcg(orow + 32 * j) : 0.0f;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float w = __shfl_sync(0xffffffffu, w_l, (c0 + c) & 31);
                    if (c0 + c < nk) {
#pragma unroll
                        for (int j = 0; j < kJ; ++j) acc[j] = fmaf(w, v[c][j], acc[j]);
                    }
                }
            }
        }
#pragma unroll
        for (int j = 0; j < kJ; ++j) {
            const size_t at = (size_t)t * d.H + rt * kTileRows + j * 32 + lane;
            if constexpr (sizeof(XT) == 4) reinterpret_cast<float*>(a.y)[at] = acc[j];
            else reinterpret_cast<__nv_bfloat16*>(a.y)[at] = __float2bfloat16_rn(acc[j]);
        }
    }
}

template <typename XT>
__device__ void i8_signaler(I8Args& a, I8Smem& S, int lane) {
    const Phases f = phases_of(a);
    volatile int* abort_flag = &S.abort_flag;
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % kSQ;
        const bool ok = wait_bar(&S.dfull[slot], (k / kSQ) & 1, abort_flag, a, 10);
        const Item r = S.done[slot];
        if (!ok || r.kind == IT_END) break;
        int last = 0;
        if (lane == 0) {
            if (r.kind == IT_PREP) {
                red_add_release(&a.ctl[kCI_Prep], 1);
            } else if (r.kind == IT_GU) {
                red_add_release(&a.ctl[i8_ctl_gu(f.nch) + r.chunk], 1);
            } else if (r.kind == IT_DOWN) {
                const int prev = atom_add_acq_rel(&a.ctl[i8_ctl_dn(f.nch) + r.rt], 1);
                // no output block can be complete before the plan is published,
                // so an unpublished plan means this was not the last tile
                const int plan = ld_acquire(&a.ctl[kCI_Plan]);
                last = plan > 0 && prev + 1 == plan - 1 + f.SC;
            }
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last && !*abort_flag) {
            signal_combine<XT>(a, r.rt, lane);
            if (a.trace && lane == 0) atomicMax(reinterpret_cast<unsigned long long*>(a.trace) + 11, globaltimer_ns());
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.dempty[slot]);
    }
}

// ------------------------------------------------------------------ consumers
template <typename XT>
__device__ __forceinline__ float2 load2(const XT* p);
template <>
__device__ __forceinline__ float2 load2<float>(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
template <>
__device__ __forceinline__ float2 load2<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Token t of x in block floating point, one 64-input group per warp at a time.
template <typename XT>
__device__ void prep_item(I8Args& a, int t, int ctid) {
    const int cw = ctid >> 5, lane = ctid & 31, G = a.d.H / kGroup;
    const XT* xr = reinterpret_cast<const XT*>(a.x) + (size_t)t * a.d.H;
    constexpr int kBatch = 12;  // groups per warp whose loads are issued together (H = 6144: all of them)
    for (int g0 = cw; g0 < G; g0 += kCW * kBatch) {
        float2 v[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int g = g0 + j * kCW;
            v[j] = g < G ? load2<XT>(xr + g * kGroup + 2 * lane) : make_float2(0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int g = g0 + j * kCW;
            if (g < G) encode_group(v[j].x, v[j].y, a.xq + ((size_t)t * G + g) * 128, a.xm + ((size_t)t * G + g) * kMetaRow,
                                    lane);
        }
    }
}

// Router rows e0, e0+1 for every token: warps 8r..8r+7 take expert e0 + r,
// each an eighth of H, with the weights held in registers across the tokens;
// the eight partial sums of a token are added in a fixed order (fp64).
template <typename XT>
__device__ void router_item(I8Args& a, I8Smem& S, double* rpart, int e0, int ctid) {
    const Dims& d = a.d;
    const int cw = ctid >> 5, lane = ctid & 31, T = a.T;
    constexpr int kParts = kCW / kRouterExperts;
    const int r = cw / kParts, part = cw % kParts;
    const int e = e0 + r;
    const int chunk = d.H / kParts;
    const XT* x = reinterpret_cast<const XT*>(a.x);
    constexpr int kV = 6;  // float4 per lane per pass: one pass for H = 6144
    for (int base = 0; base < chunk; base += kV * 128) {
        float4 wv[kV], xv0[kV];
        const float* wrow = a.wr + (size_t)(e < d.E ? e : 0) * d.H + part * chunk;
        auto load_x = [&](const XT* xr, int i) -> float4 {
            if (i >= chunk) return make_float4(0.f, 0.f, 0.f, 0.f);
            if constexpr (sizeof(XT) == 4) {
                return __ldg(reinterpret_cast<const float4*>(xr + i));
            } else {
                const uint2 u = __ldg(reinterpret_cast<const uint2*>(xr + i));
                return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                                   __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
            }
        };
        // the weights and the first token's inputs in one batch of loads (one round trip)
#pragma unroll
        for (int j = 0; j < kV; ++j) {
            const int i = base + lane * 4 + j * 128;
            wv[j] = (e < d.E && i < chunk) ? __ldg(reinterpret_cast<const float4*>(wrow + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
            xv0[j] = load_x(x + part * chunk, i);
        }
        auto store = [&](int t, double sacc) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) sacc += __shfl_xor_sync(0xffffffffu, sacc, o);
            if (lane == 0) rpart[(size_t)cw * T + t] = (base == 0 ? 0.0 : rpart[(size_t)cw * T + t]) + sacc;
        };
        {
            double sacc = 0.0;
#pragma unroll
            for (int j = 0; j < kV; ++j) {
                sacc = fma((double)wv[j].x, (double)xv0[j].x, sacc);
                sacc = fma((double)wv[j].y, (double)xv0[j].y, sacc);
                sacc = fma((double)wv[j].z, (double)xv0[j].z, sacc);
                sacc = fma((double)wv[j].w, (double)xv0[j].w, sacc);
            }
            store(0, sacc);
        }
#pragma unroll 1
        for (int t = 1; t < T; ++t) {
            const XT* xr = x + (size_t)t * d.H + part * chunk;
            double sacc = 0.0;
#pragma unroll
            for (int h2 = 0; h2 < kV; h2 += kV / 2) {  // x in two halves keeps registers bounded
                float4 xv[kV / 2];
#pragma unroll
                for (int jj = 0; jj < kV / 2; ++jj) xv[jj] = load_x(xr, base + lane * 4 + (h2 + jj) * 128);
#pragma unroll
                for (int jj = 0; jj < kV / 2; ++jj) {
                    const float4 wj = wv[h2 + jj];
                    sacc = fma((double)wj.x, (double)xv[jj].x, sacc);
                    sacc = fma((double)wj.y, (double)xv[jj].y, sacc);
                    sacc = fma((double)wj.z, (double)xv[jj].z, sacc);
                    sacc = fma((double)wj.w, (double)xv[jj].w, sacc);
                }
            }
            store(t, sacc);
        }
    }
    named_bar(1, kCT);
    for (int i = ctid; i < kRouterExperts * T; i += kCT) {
        const int rr = i / T, t = i % T, ee = e0 + rr;
        if (ee < d.E) {
            double sum = 0.0;
            for (int w = 0; w < kParts; ++w) sum += rpart[(size_t)(rr * kParts + w) * T + t];
            a.logits[(size_t)t * d.E + ee] = sum + (double)a.bias[ee];
        }
    }
}

// Exclusive scan of v over the 256 consumer threads (fixed order); returns
// the exclusive prefix and, in *total, the sum over all threads.
__device__ __forceinline__ int block_scan(int v, int ctid, int* wsum, int* total) {
    const int lane = ctid & 31, cw = ctid >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) wsum[cw] = incl;
    named_bar(1, kCT);
    int base = 0, tot = 0;
    for (int w = 0; w < kCW; ++w) {
        if (w < cw) base += wsum[w];
        tot += wsum[w];
    }
    named_bar(1, kCT);
    *total = tot;
    return base + incl - v;
}

// Top-k of the T tokens and the batch-union plan, by the consumers of the CTA
// that finished the last router item. Everything is stored before the one
// release of the plan flag (1 + number of routed chunks).
__device__ void consumer_plan(I8Args& a, I8Smem& S, uint8_t* scratch, int ctid) {
    const Dims& d = a.d;
    const int T = a.T, E = d.E, K = d.K, TK = T * K;
    const int cw = ctid >> 5, lane = ctid & 31;
    int* sids = reinterpret_cast<int*>(scratch);           // [TK]
    float* sw = reinterpret_cast<float*>(sids + TK);       // [TK]
    int* scnt = reinterpret_cast<int*>(sw + TK);           // [E]
    int* soff = scnt + E;                                  // [E]
    if (a.trace && ctid == 0) a.trace[4] = (long long)globaltimer_ns();
    if (a.given_ids) {  // routing computed before the launch
        for (int sl = ctid; sl < TK; sl += kCT) {
            sids[sl] = __ldcg(a.given_ids + sl);
            sw[sl] = __ldcg(a.given_w + sl);
        }
    } else {
        for (int t = cw; t < T; t += kCW) {
            int id;
            float wt;
            if (E <= 256) warp_topk8<true>(a.logits + (size_t)t * E, E, K, a.topp, lane, &id, &wt);
            else warp_topk<true>(a.logits + (size_t)t * E, E, K, a.topp, lane, &id, &wt);
            if (lane < K) {
                sids[t * K + lane] = (id >= a.ep_lo && id < a.ep_hi) ? id : -1;
                sw[t * K + lane] = wt;
            }
        }
    }
    for (int e = ctid; e < E; e += kCT) scnt[e] = 0;
    named_bar(1, kCT);
    if (a.trace && ctid == 0) a.trace[5] = (long long)globaltimer_ns();
    for (int sl = ctid; sl < TK; sl += kCT)
        if (sids[sl] >= 0) atomicAdd(&scnt[sids[sl]], 1);  // < 0: an empty slot
    named_bar(1, kCT);
    // per expert: first position, distinct-expert rank, first chunk
    unsigned long long* entries = entries_of(a, d.S * a.cps + a.ncmax);
    int carry = 0, ucarry = 0, ccarry = 0;
    for (int c0 = 0; c0 < E; c0 += kCT) {
        const int e = c0 + ctid;
        const int c = e < E ? scnt[e] : 0;
        const int f = c > 0, nchk = (c + a.ntc - 1) / a.ntc;
        int tot, utot, ctot;
        const int off = carry + block_scan(c, ctid, S.wsum, &tot);
        const int rank = ucarry + block_scan(f, ctid, S.wsum, &utot);
        const int ch0 = ccarry + block_scan(nchk, ctid, S.wsum, &ctot);
        if (e < E) {
            if (f) a.p.unique[rank] = e;
            for (int i = 0; i < nchk; ++i) {
                const unsigned long long v = (1ull << 63) | (unsigned long long)e |
                                             ((unsigned long long)(off + i * a.ntc) << 16) |
                                             ((unsigned long long)min(a.ntc, c - i * a.ntc) << 36);
                entries[ch0 + i] = v;
            }
            a.p.off[e] = off;
            a.p.cnt[e] = c;
            soff[e] = off;
        }
        carry += tot;
        ucarry += utot;
        ccarry += ctot;
    }
    if (a.trace && ctid == 0) a.trace[6] = (long long)globaltimer_ns();
    named_bar(1, kCT);
    // slot (t, k): position = first position of its expert + earlier tokens of that expert
    for (int sl = ctid; sl < TK; sl += kCT) {
        const int e = sids[sl], t = sl / K;
        a.p.ids[sl] = e;
        a.p.w[sl] = sw[sl];
        if (e < 0) {
            a.p.pos[sl] = -1;
            continue;
        }
        int rank = 0;
        for (int s2 = 0; s2 < t * K; ++s2) rank += sids[s2] == e;
        const int q = soff[e] + rank;
        a.p.pos[sl] = q;
        a.p.tok[q] = t;
    }
    for (int i = ctid; i < d.S * T; i += kCT) a.p.tok[TK + i] = i % T;
    if (ctid == 0) {
        a.p.off[E] = carry;
        *a.p.n_unique = ucarry;
        *a.p.n_active = ucarry + d.S;
    }
    if (a.trace && ctid == 0) a.trace[7] = (long long)globaltimer_ns();
    if (ctid == 0) S.plan_chunks = ccarry;
    named_bar(1, kCT);  // orders every consumer's plan writes before thread 0's release
    if (ctid == 0) {
        if (a.trace) a.trace[8] = (long long)globaltimer_ns();
        st_release(&a.ctl[kCI_Plan], ccarry + 1);
        if (a.trace) a.trace[3] = (long long)globaltimer_ns();
    }
}

// One 64-input block of one 16-row sub-tile for nch column chunks (4 tokens
// each): the lane's 32 weights (16 bytes of nibbles), its rows' fp16 scales,
// and per chunk the B fragment and the group meta of its token.
template <int NCH>
__device__ __forceinline__ void block_mma(const uint8_t* bp, const uint8_t* blimb, const uint8_t* bmeta, int g, int G,
                                          int sub, int lane, int nt, float (&acc)[2][2]) {
    const int gi = lane >> 2, t4 = lane & 3;
    const uint4 w = *reinterpret_cast<const uint4*>(bp + sub * 512 + lane_slot(lane) * 16);
    const uint32_t sv = *reinterpret_cast<const uint32_t*>(bp + kNibbleBytes + sub * 32 + gi * 4);
    // offset-binary codes v = q + 8 of rows gi (low nibbles) and gi+8 (high nibbles, as 16 v)
    const uint32_t a0 = w.x & 0x0F0F0F0Fu, a1 = w.x & 0xF0F0F0F0u, a2 = w.y & 0x0F0F0F0Fu, a3 = w.y & 0xF0F0F0F0u;
    const uint32_t a4 = w.z & 0x0F0F0F0Fu, a5 = w.z & 0xF0F0F0F0u, a6 = w.w & 0x0F0F0F0Fu, a7 = w.w & 0xF0F0F0F0u;
    const float2 sc = __half22float2(*reinterpret_cast<const __half2*>(&sv));
    const float s0 = sc.x, s1 = sc.y * 0.0625f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
        // B column gi: token 4c + gi/2 of the item, part gi%2 (hi, lo)
        // columns of absent tokens are not read (zero): fewer shared-memory wavefronts
        uint4 bf = make_uint4(0u, 0u, 0u, 0u);
        int4 mt = make_int4(0, 0, 0, 0);
        if (c * kChunkTok + (gi >> 1) < nt)
            bf = *reinterpret_cast<const uint4*>(blimb + ((size_t)(c * kChunkTok + (gi >> 1)) * G + g) * 128 +
                                                 (gi & 1) * 64 + t4 * 16);
        if (c * kChunkTok + t4 < nt)
            mt = *reinterpret_cast<const int4*>(bmeta + (size_t)(c * kChunkTok + t4) * meta_slot_bytes(G) +
                                                (size_t)g * kMetaRow);
        // one accumulator starts at the nibble offset's correction, -8 sum(part) (x16 for
        // rows gi+8); the two 32-input halves accumulate separately (no dependency)
        int cc[4] = {mt.y, mt.z, mt.y * 16, mt.z * 16};
        int cd[4] = {0, 0};
        mma_u8s8(cc, a0, a1, a2, a3, bf.x, bf.y);
        mma_u8s8(cd, a4, a5, a6, a7, bf.z, bf.w);
        const float sx = __int_as_float(mt.x);
        const int p0 = (cc[0] + cd[0]) * 256 + (cc[1] + cd[1]), p1 = (cc[2] + cd[2]) * 256 + (cc[3] + cd[3]);
        acc[c][0] = fmaf(s0 * sx, (float)p0, acc[c][0]);  // row gi,   token 4c + t4
        acc[c][1] = fmaf(s1 * sx, (float)p1, acc[c][1]);  // row gi+8, token 4c + t4
    }
}

template <typename XT>
__device__ void weight_item(I8Args& a, I8Smem& S, const Item& it, uint32_t q, uint8_t* ring, uint8_t* barea,
                            uint32_t& slot_s, uint32_t& phase_s, int ctid) {
    const Dims& d = a.d;
    const Phases f = phases_of(a);
    const int cw = ctid >> 5, lane = ctid & 31, gi = lane >> 2, t4 = lane & 3;
    const bool gu = it.kind == IT_GU;
    const int G = gu ? f.Ggu : f.Gd;
    const int nt = it.cnt;
    volatile int* abort_flag = &S.abort_flag;

    uint8_t* blimb = buf_limbs(a, barea, 0);
    uint8_t* bmeta = buf_meta(a, barea, 0);
    bool have;  // the B operands are in place (false only after an abort)
    if (a.nbuf == 2) {
        // ---- two B buffers: the operands are in the buffer of the item's queue slot, staged
        // by the producer when it published the item, else by consumer 0 now
        const int k = (int)(q % kQ);
        const uint32_t par = (q / kQ) & 1;
        blimb = buf_limbs(a, barea, k);
        bmeta = buf_meta(a, barea, k);
        if (!it.staged) {  // uniform: every consumer read the same item
            if (ctid == 0) {
                bool ok;
                if (gu) ok = wait_geq(&a.ctl[kCI_Prep], f.P, abort_flag, a, 5);
                else ok = it.ready || wait_geq(&a.ctl[i8_ctl_gu(f.nch) + it.chunk], f.RTgu, abort_flag, a, 6);
                // testing aid: the launch's first gate/up tile waits on a flag that nothing sets
                if (ok && a.wait_test && gu && it.chunk == 0 && it.rt == 0)
                    wait_geq(&a.ctl[kCI_Never], 1, abort_flag, a, 99);
                if (!*abort_flag) stage_slot(a, S, it, k, par, barea);
            }
            named_bar(1, kCT);
        }
        have = wait_bar(&S.bslot_full[k], par, abort_flag, a, 8);
        if (ctid == 0 && have) S.bslot_pending[k] = 0;
    } else {
        // ---- the item's tokens as B operands (staged once, reused by items with the same tokens)
        bool same;
        if (gu) {
            same = S.staged_kind == IT_GU && S.staged_n == nt;
            for (int i = 0; same && i < nt; ++i) {
                same = S.staged_tok[i] == item_token(a, it, i);
            }
        } else {
            same = S.staged_kind == IT_DOWN && S.staged_key == it.chunk;
        }
        named_bar(1, kCT);  // every consumer has read the staging record before it changes
        if (!same) {  // uniform: every consumer read the same shared values
            if (ctid == 0) {
                bool ok;
                if (gu) ok = wait_geq(&a.ctl[kCI_Prep], f.P, abort_flag, a, 5);
                else ok = it.ready || wait_geq(&a.ctl[i8_ctl_gu(f.nch) + it.chunk], f.RTgu, abort_flag, a, 6);
                // testing aid: the launch's first gate/up tile waits on a flag that nothing sets
                if (ok && a.wait_test && gu && it.chunk == 0 && it.rt == 0)
                    wait_geq(&a.ctl[kCI_Never], 1, abort_flag, a, 99);
                if (!*abort_flag) {
                    fence_proxy_async_global();
                    const uint32_t lbytes = (uint32_t)G * 128, mbytes = (uint32_t)G * kMetaRow;
                    mbar_arrive_expect_tx(&S.bfull, (uint32_t)nt * (lbytes + mbytes));
                    S.bpending = 1;
                    if (gu) {
                        for (int i = 0; i < nt; ++i) {
                            const int tok = item_token(a, it, i);
                            S.staged_tok[i] = tok;
                            bulk_g2s(blimb + (size_t)i * lbytes, a.xq + (size_t)tok * lbytes, lbytes, &S.bfull);
                            bulk_g2s(bmeta + (size_t)i * meta_slot_bytes(G), a.xm + (size_t)tok * mbytes, mbytes, &S.bfull);
                        }
                    } else {
                        bulk_g2s(blimb, a.hq + (size_t)it.pos * lbytes, nt * lbytes, &S.bfull);
                        for (int i = 0; i < nt; ++i)
                            bulk_g2s(bmeta + (size_t)i * meta_slot_bytes(G), a.hm + (size_t)(it.pos + i) * mbytes, mbytes,
                                     &S.bfull);
                    }
                    S.staged_kind = it.kind;
                    S.staged_n = nt;
                    S.staged_key = it.chunk;
                } else {
                    S.staged_kind = -1;
                }
            }
            named_bar(1, kCT);
            bool landed = true;
            if (S.staged_kind == it.kind) landed = wait_bar(&S.bfull, S.bphase & 1, abort_flag, a, 8);
            named_bar(1, kCT);
            if (ctid == 0 && S.staged_kind == it.kind && landed) {
                ++S.bphase;
                S.bpending = 0;
            }
        }
        have = S.staged_kind == it.kind;
    }

    // ---- stream the weight tile through the ring
    if (a.trace && ctid == 0) S.t_loop0 = globaltimer_ns();
    float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const int sub = cw % kSub, half = cw / kSub;  // warps sub and sub + 8 (two per sub-tile) share a sub-tile
    const uint32_t stage_bytes = (uint32_t)a.sb * kBlockBytes;
    const int nst = (G + a.sb - 1) / a.sb;
    const int nch = (nt + kChunkTok - 1) / kChunkTok;
    bool seen = false;  // this thread saw the stage complete while working on the previous one
    for (int i = 0; i < nst; ++i) {
        uint64_t tw = 0;
        if (a.trace && ctid == 0) tw = globaltimer_ns();
        const bool ok = seen || wait_bar(&S.full[slot_s], phase_s, abort_flag, a, 7);
        // test the next stage now (non-blocking); the answer is used after this stage's groups
        bool next_full = false;
        if (i + 1 < nst) {
            const uint32_t ns = slot_s + 1 == (uint32_t)a.nstages ? 0 : slot_s + 1;
            next_full = mbar_test_wait(&S.full[ns], ns == 0 ? phase_s ^ 1 : phase_s);
        }
        if (a.trace && ctid == 0) {
            const uint64_t dw = globaltimer_ns() - tw;
            if (i == 0) S.first_wait_ns = dw;
            S.total_wait_ns += dw;
        }
        if (ok && have) {
            const uint8_t* stage = ring + (size_t)slot_s * stage_bytes;
            const int g0 = i * a.sb;
            const int nb = min(a.sb, G - g0);
            if (nch == 1) {
#pragma unroll 4
                for (int bb = half; bb < nb; bb += kWS)
                    block_mma<1>(stage + bb * kBlockBytes, blimb, bmeta, g0 + bb, G, sub, lane, nt, acc);
            } else {
#pragma unroll 2
                for (int bb = half; bb < nb; bb += kWS)
                    block_mma<2>(stage + bb * kBlockBytes, blimb, bmeta, g0 + bb, G, sub, lane, nt, acc);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot_s]);
        if (++slot_s == (uint32_t)a.nstages) { slot_s = 0; phase_s ^= 1; }
        seen = next_full;
    }
    if (half == 1) *reinterpret_cast<float4*>(S.accx[sub][lane]) = make_float4(acc[0][0], acc[0][1], acc[1][0], acc[1][1]);
    if (a.trace && ctid == 0) S.t_loop1 = globaltimer_ns();
    if (ctid == 0) S.aborted = *abort_flag;
    named_bar(1, kCT);
    const bool aborted = S.aborted != 0;  // uniform: read after the barrier
    if (aborted) return;
    const bool lead = half == 0;  // the first warp of each sub-tile finishes the item
    if (kWS == 2 && lead) {  // fixed order: blocks of the first warp, then those of the second
        const float4 o = *reinterpret_cast<const float4*>(S.accx[sub][lane]);
        acc[0][0] += o.x; acc[0][1] += o.y; acc[1][0] += o.z; acc[1][1] += o.w;
    }

    // ---- epilogue: lane (gi, t4) holds rows gi, gi+8 of sub-tile `sub` for tokens t4 and 4 + t4
    if (!gu) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int i = c * kChunkTok + t4;
            if (lead && c < nch && i < nt) {
                const int r0 = it.rt * kTileRows + sub * kSubRows + gi;
                float* orow = a.o + (size_t)(it.pos + i) * d.H;
                orow[r0] = acc[c][0];
                orow[r0 + 8] = acc[c][1];
            }
        }
        return;
    }
    // gate/up: row gi is gate row j, row gi+8 the up row j of the same j; h[j] for the
    // item's tokens, then h of down's input group g = rt (h indices 64 rt .. 64 rt + 63,
    // index k = 8 sub + gi within it) in block floating point, as encode_group does
    float hv[2] = {0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        if (lead && c < nch && c * kChunkTok + t4 < nt) hv[c] = silu_f(acc[c][0]) * acc[c][1];
        float m = fabsf(hv[c]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (lead && gi == 0) S.hmaxw[sub][c * kChunkTok + t4] = m;
    }
    named_bar(1, kCT);
    const int k = sub * 8 + gi;
    const int g = it.rt;
    int hs[2][2] = {{0, 0}, {0, 0}};
    float sxv[2] = {0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 2; ++c) {
        const int i = c * kChunkTok + t4;
        if (lead && c < nch && i < nt) {
            float m = 0.0f;
            for (int w = 0; w < kSub; ++w) m = fmaxf(m, S.hmaxw[w][i]);
            const int e = group_exponent(m);
            const int xi = __float2int_rn(hv[c] * pow2f(e));
            const int hi = (xi + 128) >> 8, lo = xi - 256 * hi;
            uint8_t* dst = a.hq + ((size_t)(it.pos + i) * f.Gd + g) * 128;
            dst[limb_offset(k)] = (uint8_t)(int8_t)hi;
            dst[64 + limb_offset(k)] = (uint8_t)(int8_t)lo;
            hs[c][0] = hi;
            hs[c][1] = lo;
            sxv[c] = pow2f(-e);
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            hs[c][0] += __shfl_xor_sync(0xffffffffu, hs[c][0], o);
            hs[c][1] += __shfl_xor_sync(0xffffffffu, hs[c][1], o);
        }
        if (lead && gi == 0) {
            S.hsum[sub][c * kChunkTok + t4][0] = hs[c][0];
            S.hsum[sub][c * kChunkTok + t4][1] = hs[c][1];
        }
    }
    named_bar(1, kCT);
    if (cw == 0 && gi == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            const int i = c * kChunkTok + t4;
            if (c < nch && i < nt) {
                int sh = 0, sl = 0;
                for (int w = 0; w < kSub; ++w) { sh += S.hsum[w][i][0]; sl += S.hsum[w][i][1]; }
                *reinterpret_cast<int4*>(a.hm + ((size_t)(it.pos + i) * f.Gd + g) * 16) =
                    make_int4(__float_as_int(sxv[c]), -8 * sh, -8 * sl, 0);
            }
        }
    }
}

// Bytes of the B area (token limbs and meta of one item; also the scratch of
// router items and of the plan).
__host__ __device__ inline size_t b_area_bytes(const Dims& d, int T, int ntc) {
    const int G = (d.H > d.I ? d.H : d.I) / kGroup;
    const size_t operands = (size_t)ntc * ((size_t)G * 128 + meta_slot_bytes(G));
    const size_t plan = (size_t)T * d.K * 8 + (size_t)2 * d.E * 4;
    const size_t router = (size_t)kCW * T * 8;
    size_t m = operands > plan ? operands : plan;
    return m > router ? m : router;
}

__host__ __device__ inline size_t head_bytes() { return (sizeof(I8Smem) + 127) & ~(size_t)127; }

template <typename XT>
__global__ void __launch_bounds__(kFT, 1) moe_decode_i8_kernel(I8Args a) {
    extern __shared__ __align__(128) uint8_t smem[];
    I8Smem& S = *reinterpret_cast<I8Smem*>(smem);
    uint8_t* ring = smem + head_bytes();
    uint8_t* barea = ring + (size_t)a.nstages * a.sb * kBlockBytes;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < a.nstages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], kCW); }
        for (int i = 0; i < kQ; ++i) { mbar_init(&S.qfull[i], 1); mbar_init(&S.qempty[i], 1); }
        for (int i = 0; i < kSQ; ++i) { mbar_init(&S.dfull[i], kCT); mbar_init(&S.dempty[i], 1); }
        mbar_init(&S.bfull, 1);
        for (int i = 0; i < kQ; ++i) {
            mbar_init(&S.bslot_full[i], 1);
            S.bslot_pending[i] = 0;
        }
        S.abort_flag = 0;
        S.bphase = 0;
        S.bpending = 0;
        S.aborted = 0;
        S.staged_kind = -1;
        S.staged_n = -1;
        mbar_fence_init();
        if (a.trace) atomicMin(reinterpret_cast<unsigned long long*>(a.trace) + 9, globaltimer_ns());
    }
    __syncthreads();
    if (warp == kProducerWarp) {
        if (lane == 0) i8_producer(a, S, ring);
        __syncwarp();
    } else if (warp == kSignalWarp) {
        i8_signaler<XT>(a, S, lane);
    } else {
        const int ctid = tid;
        uint32_t q = 0, slot_s = 0, phase_s = 0;
        for (uint32_t k = 0;; ++k) {
            // thread 0 takes the next item and publishes it, so every consumer
            // thread takes the same branch below
            const uint32_t slot = q % kQ;
            if (ctid == 0) {
                const bool ok = wait_bar(&S.qfull[slot], (q / kQ) & 1, &S.abort_flag, a, 9);
                S.cur[q & 1] = S.items[slot];
                if (!ok || S.abort_flag) S.cur[q & 1].kind = IT_END;
            }
            named_bar(1, kCT);
            const Item it = S.cur[q & 1];
            const uint64_t t_begin = (a.trace && ctid == 0) ? globaltimer_ns() : 0;
            if (ctid == 0) S.first_wait_ns = S.total_wait_ns = S.t_loop0 = S.t_loop1 = 0;
            if (it.kind == IT_PREP || it.kind == IT_ROUTER) {
                // the CTA that finishes the last router item (with the routing
                // given: the last quantisation item) builds the plan
                if (it.kind == IT_PREP) {
                    prep_item<XT>(a, it.ex, ctid);
                } else {
                    if (ctid == 0) S.staged_kind = -1;  // the B area becomes scratch
                    router_item<XT>(a, S, reinterpret_cast<double*>(barea), it.ex, ctid);
                }
                const bool counted = it.kind == IT_ROUTER || a.given_ids;
                if (counted) {
                    named_bar(1, kCT);
                    if (ctid == 0) {
                        const int n_items = it.kind == IT_ROUTER ? (a.d.E + kRouterExperts - 1) / kRouterExperts : a.T;
                        const uint64_t t0 = a.trace ? globaltimer_ns() : 0;
                        // the barrier orders the other consumers' logits before this
                        // release, which carries them to the plan builders (cumulative)
                        S.last = atom_add_acq_rel(&a.ctl[kCI_Router], 1) == n_items - 1;
                        if (S.last) S.staged_kind = -1;  // the B area becomes the plan's scratch
                        if (S.last && a.trace) { a.trace[1] = (long long)t0; a.trace[2] = (long long)globaltimer_ns(); }
                    }
                    named_bar(1, kCT);
                    if (S.last) {  // uniform: S.last is read after the barrier
                        consumer_plan(a, S, barea, ctid);
                        // no routed chunk and no shared expert (a rank of an expert-parallel layer
                        // that holds none of the batch's experts): no down item will combine the
                        // output, so it is the residual (or 0) here
                        if (S.plan_chunks == 0 && a.d.S == 0) {
                            for (size_t i = ctid; i < (size_t)a.T * a.d.H; i += kCT) {
                                const float v = a.residual ? a.residual[i] : 0.0f;
                                if constexpr (sizeof(XT) == 4) reinterpret_cast<float*>(a.y)[i] = v;
                                else reinterpret_cast<__nv_bfloat16*>(a.y)[i] = __float2bfloat16_rn(v);
                            }
                        }
                    }
                }
            } else if (it.kind == IT_GU || it.kind == IT_DOWN) {
                weight_item<XT>(a, S, it, q, ring, barea, slot_s, phase_s, ctid);
            }
            // hand the completion to the signaler: the record first, then every
            // consumer thread arrives after its own global writes
            const uint32_t ds = k % kSQ;
            if (ctid == 0) {
                if (k >= kSQ) wait_bar(&S.dempty[ds], ((k / kSQ) - 1) & 1, &S.abort_flag, a, 11);
                S.done[ds] = it;
            }
            // every consumer's writes precede its arrival (release, CTA scope); the
            // signaler's release atomic that follows carries them to other CTAs
            named_bar(1, kCT);
            mbar_arrive(&S.dfull[ds]);
            if (a.trace && ctid == 0 && it.kind != IT_END) {
                const unsigned long long r = atomicAdd(reinterpret_cast<unsigned long long*>(a.trace), 1ull);
                if (r < (unsigned long long)a.trace_cap) {
                    long long* rec = a.trace + 16 + 8 * r;
                    const int kind = it.kind == IT_ROUTER ? 1 : it.kind == IT_GU ? 2 : it.kind == IT_DOWN ? 3 : 4;
                    rec[0] = ((long long)blockIdx.x << 40) | ((long long)kind << 32) | ((long long)(it.ex & 0xFFFF) << 16) |
                             (it.rt & 0xFFFF);
                    rec[1] = (long long)t_begin;
                    rec[2] = (long long)globaltimer_ns();
                    rec[3] = (long long)S.first_wait_ns;
                    rec[4] = it.cnt;
                    rec[5] = (long long)S.total_wait_ns;
                    rec[6] = (long long)S.t_loop0;
                    rec[7] = (long long)S.t_loop1;
                }
            }
            if (ctid == 0 && it.kind != IT_END) mbar_arrive(&S.qempty[slot]);
            ++q;
            if (it.kind == IT_END) break;
        }
    }
    __syncthreads();
    if (tid == 0) {
        // a B staging still in flight (after an abort) must land before the CTA exits
        if (S.bpending) {
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&S.bfull, S.bphase & 1) && globaltimer_ns() - t0 < (uint64_t)a.wait_ns) {
            }
        }
        for (int i = 0; i < kQ; ++i) {
            if (!S.bslot_pending[i]) continue;
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&S.bslot_full[i], S.bslot_parity[i]) && globaltimer_ns() - t0 < (uint64_t)a.wait_ns) {
            }
        }
        __threadfence();
        S.last = atomicAdd(&a.ctl[kCI_Exit], 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (S.last) {
        // last CTA out: clear the control block for the next launch (keep the error)
        if (a.trace && tid == 0) a.trace[10] = (long long)globaltimer_ns();
        __threadfence();
        const int n = i8_ctl_ints(a.d.S * a.cps + a.ncmax, a.d.H, a.ncmax);
        for (int i = tid; i < n; i += blockDim.x)
            if (i != kCI_Error) a.ctl[i] = 0;
        __threadfence();
    }
}

size_t i8_smem_bytes(const Dims& d, int T, int ntc, int nstages, int sb) {
    return head_bytes() + (size_t)nstages * sb * kBlockBytes + b_area_bytes(d, T, ntc);
}

}  // namespace

// Routed chunks of a launch at most: every distinct expert has one chunk more
// than its full chunks of ntc tokens.
int i8_ncmax(const Dims& d, int T, int ntc) {
    const int TK = T * d.K;
    return (TK < d.E ? TK : d.E) + TK / ntc;
}

int i8_ctl_ints_for(const Dims& d, int T) {
    // the layout with 4-token items bounds every launch of up to T tokens
    const int ncmax = i8_ncmax(d, T, 4);
    return i8_ctl_ints(d.S * ((T + 3) / 4) + ncmax, d.H, ncmax);
}

// Ring geometry and item size for T tokens. Four-token items leave room for
// the largest copies (two stages of up to 16 blocks, 69,632 bytes each: fewer
// stage hand-offs per block); eight-token items stream a hot expert's weights
// half as often but fit only smaller copies (three stages of 8 blocks). On a
// B200 the first is faster up to 32 tokens, the second at 64 (Zipf routing).
bool i8_geometry(const Dims& d, int T, size_t smem_limit, int max_stages, int max_sb, int* ntc, int* nstages, int* sb) {
    const int order[2] = {T > 32 ? 8 : 4, T > 32 ? 4 : (T > 4 ? 8 : 4)};
    for (int nt : order) {
        for (int b = max_sb; b >= 2; b -= 2) {
            int ns = max_stages < kMaxStages ? max_stages : kMaxStages;
            while (ns > 0 && i8_smem_bytes(d, T, nt, ns, b) > smem_limit) --ns;
            const int need = nt == 8 ? 3 : 2;
            if (ns >= need) { *ntc = nt; *nstages = ns; *sb = b; return true; }
        }
    }
    return false;
}

template <typename XT>
static cudaError_t launch_i8_t(const I8Args& a, int n_sm, size_t smem_limit, cudaStream_t st) {
    static int configured_device = -1;  // the opt-in limit is set once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(moe_decode_i8_kernel<XT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem_limit);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const size_t smem = i8_smem_bytes(a.d, a.T, a.ntc, a.nstages, a.sb);
    moe_decode_i8_kernel<XT><<<n_sm, kFT, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode_i8(const I8Launch& l, cudaStream_t st) {
    if (l.T < 1 || l.T > kI8MaxTok || l.T * l.d.K > kI8MaxSlots) return cudaErrorInvalidValue;
    I8Args a;
    a.weights = l.weights; a.d = l.d; a.wr = l.wr; a.bias = l.bias; a.x = l.x; a.y = l.y; a.residual = l.residual;
    a.T = l.T; a.p = l.p; a.logits = l.logits; a.given_ids = l.given_ids; a.given_w = l.given_w; a.topp = l.topp; a.ep_lo = l.ep_lo; a.ep_hi = l.ep_hi > 0 ? l.ep_hi : l.d.E; a.xq = l.xq; a.xm = l.xm; a.hq = l.hq; a.hm = l.hm; a.o = l.o;
    a.ctl = l.ctl; a.trace = l.trace; a.trace_cap = l.trace_cap;
    a.wait_ns = l.wait_ns > 0 ? l.wait_ns : 1000000000ll;
    a.wait_test = l.wait_test;
    if (!i8_geometry(l.d, l.T, l.smem_limit, l.max_stages, l.max_sb, &a.ntc, &a.nstages, &a.sb))
        return cudaErrorInvalidConfiguration;
    a.cps = (l.T + a.ntc - 1) / a.ntc;
    // two B buffers (the next item's operands staged by the producer while the current
    // item streams) when two of the largest chunks fit in the area sized for ntc positions.
    // A chunk holds distinct tokens, so at most T positions, except under expert top-p,
    // where a token's dropped slots repeat its first expert (weight 0): up to T K.
    const bool topp_on = l.topp > 0.0 && l.topp < 1.0;  // the top-k's own test
    const int span = topp_on ? l.T * l.d.K : l.T;
    const int maxchunk = span < a.ntc ? span : a.ntc;
    a.nbuf = 2 * maxchunk <= a.ntc ? 2 : 1;
    a.nbt = a.nbuf == 2 ? maxchunk : a.ntc;
    a.ncmax = i8_ncmax(l.d, l.T, a.ntc);
    if (l.dt == COLI_F32) return launch_i8_t<float>(a, l.n_sm, l.smem_limit, st);
    return launch_i8_t<__nv_bfloat16>(a, l.n_sm, l.smem_limit, st);
}

bool decode_i8_supported(const Dims& d, int T, size_t smem_limit) {
    int ntc, ns, sb;
    return T >= 1 && T <= kI8MaxTok && T * d.K <= kI8MaxSlots && i8_geometry(d, T, smem_limit, kMaxStages, kMaxSB, &ntc, &ns, &sb);
}

}  // namespace coli
