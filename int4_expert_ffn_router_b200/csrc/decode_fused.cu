// decode_fused.cu -- the whole MoE layer for a few tokens in one persistent
// kernel: router, top-k, batch-union plan, fused int4 gate/up + SwiGLU,
// down, and the weighted combine with the shared expert.
//
// Decode streams each active expert's ~20 MB once ("Colibri: 2400 lines of
// pure C ...", kechuai.cn, section 二: one read per unique expert per batch,
// the three matrices adjacent), so the kernel is HBM-bound: it must keep
// enough bytes in flight and keep global-memory round trips (about 1-2 us
// each while HBM is saturated) off the path of the warps that do the math.
// One CTA per SM, three warp roles:
//  * a producer warp takes work tickets and streams each item's weight tile
//    into a shared-memory ring with bulk asynchronous copies (the TMA engine)
//    of up to 34,816 bytes, completing on mbarriers;
//  * eight consumer warps (one 16-row sub-tile each) dequantise int4 to
//    exact fp16 and multiply on the tensor cores from registers
//    (int4_mma.cuh): for a decode GEMV the CUDA-core instruction budget per
//    streamed weight, not the tensor pipe, is the limit;
//  * a signaler warp publishes completions (release atomics), builds the
//    top-k and the batch-union plan when the last router item lands, and
//    combines each 128-row block of y when its last down tile lands, so the
//    consumers never wait on a global round trip to hand work off.
// Tickets are handed out in dependency order: router rows, shared-expert
// gate/up, routed gate/up, shared-expert down, routed down. An item only
// waits for items with smaller tickets, which running CTAs already hold, so
// the schedule cannot deadlock; every wait is bounded in time and reports a
// timeout through the control block instead of hanging.
#include "common.cuh"
#include "int4_mma.cuh"
#include "kernels.cuh"
#include "topk.cuh"

namespace coli {

constexpr int kCW = 8;                       // consumer warps (one 16-row sub-tile each)
constexpr int kCT = kCW * 32;                // consumer threads
constexpr int kProducerWarp = kCW;
constexpr int kSignalWarp = kCW + 1;
constexpr int kFT = (kCW + 2) * 32;          // all threads
constexpr int kMaxSB = 8;                    // 4352-byte blocks per ring stage (at most)
constexpr int kQ = 2;                        // item queue slots (lookahead of one item)
constexpr int kSQ = 4;                       // completion records in flight to the signaler
constexpr uint64_t kWaitNs = 1000000000ull;  // every wait gives up after 1 s
constexpr int kRouterExperts = 2;            // experts per router item (4 warps each)

enum { IT_END = 0, IT_ROUTER = 1, IT_GU = 2, IT_DOWN = 3 };

struct Item {
    int kind, ex, rt, off, cnt;
    int tokens;  // gate/up: token ids, 8 bits each, ascending
    int ready;   // down: gate/up of `ex` already complete when published
    int pad;
    long long pushed_ns;  // trace only
};

struct FusedArgs {
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
    float* h;
    float* o;
    int* ctl;
    int umax;     // min(T*K, E): upper bound of distinct routed experts
    int nstages;  // ring stages
    int sb;       // 4352-byte blocks per stage; the bulk copies are sb * 4352 bytes
    long long* trace;  // item timeline (NULL: off)
    int trace_cap;
};

struct FusedSmem {
    uint64_t full[kMaxStages], empty[kMaxStages], qfull[kQ], qempty[kQ], dfull[kSQ], dempty[kSQ];
    Item items[kQ];
    Item cur[2];
    Item done[kSQ];
    int abort_flag;
    int last;
    int staged_n, staged_rows[kFusedMaxTok];
    float xscale[kFusedMaxTok];
    float mred[(kCW + 1) * kFusedMaxTok];
    double rpart[kCW][kFusedMaxTok];
    int sids[kFusedMaxTok * 32];
    float sw[kFusedMaxTok * 32];
    int wsum[kCW], wflag[kCW];
    unsigned long long first_wait_ns, total_wait_ns;
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

__device__ __forceinline__ void red_max_u32(unsigned* p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void set_error(FusedArgs& a, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    atomicCAS(&a.ctl[kCtlError], 0, code);
}

// Bounded wait on an mbarrier phase; gives up when the CTA aborts or after kWaitNs.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort_flag, FusedArgs& a,
                                         int code) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            set_error(a, abort_flag, code);
            return false;
        }
    }
}

// Bounded wait until *p >= target (acquire).
__device__ __forceinline__ bool wait_geq(const int* p, int target, volatile int* abort_flag, FusedArgs& a, int code) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (ld_acquire(p) >= target) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > kWaitNs) {
            set_error(a, abort_flag, code);
            return false;
        }
        __nanosleep(64);
    }
}

// Running max |h| of each position (float bits; non-negative floats order as
// unsigned integers), after the tile counters in the control block.
__device__ __forceinline__ unsigned* hmax_of(FusedArgs& a) {
    return reinterpret_cast<unsigned*>(a.ctl + ctl_hmax_at(a.d.E, a.d.S, a.d.H));
}

// Packed plan entries: bit 63 valid, [0,16) expert, [16,32) first position,
// [32,40) tokens, [40,48) token ids (2 bits each, ascending).
__device__ __forceinline__ unsigned long long* entries_of(FusedArgs& a) {
    return reinterpret_cast<unsigned long long*>(a.ctl + ctl_entries_at(a.d.E, a.d.S, a.d.H, a.d.K));
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ------------------------------------------------------------------ producer
__device__ void fused_producer(FusedArgs& a, FusedSmem& S, uint8_t* ring) {
    const Dims& d = a.d;
    const int T = a.T;
    const int RTgu = 2 * d.I / kTileRows, RTd = d.H / kTileRows;
    const int Ggu = d.H / kGroup, Gd = d.I / kGroup;
    const int n_router = (d.E + kRouterExperts - 1) / kRouterExperts;
    // ticket ranges: router | shared gate/up | routed gate/up | shared down | routed down
    const int t_sg = n_router, t_ug = t_sg + d.S * RTgu, t_sd = t_ug + a.umax * RTgu;
    const int t_ud = t_sd + d.S * RTd, t_end = t_ud + a.umax * RTd;
    int all_tokens = 0;
    for (int t = 0; t < T; ++t) all_tokens |= t << (8 * t);
    volatile int* abort_flag = &S.abort_flag;
    const unsigned long long* entries = entries_of(a);
    uint32_t q = 0, gs = 0, slot_s = 0, phase_s = 0;
    bool first_ticket = true;
    while (true) {
        Item it{IT_END, 0, 0, 0, 0, 0, 0, 0, 0};
        if (!*abort_flag) {
            // the first ticket of CTA b is b (no contended atomic at start-up); later ones
            // come from the shared counter, after the gridDim.x static ones
            const int t = first_ticket ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(&a.ctl[kCtlTicket], 1);
            first_ticket = false;
            const bool routed = (t >= t_ug && t < t_sd) || (t >= t_ud && t < t_end);
            if (t < t_sg) {
                it.kind = IT_ROUTER;
                it.ex = t * kRouterExperts;
            } else if (t < t_ug) {
                const int j = (t - t_sg) / RTgu;
                it = Item{IT_GU, d.E + j, (t - t_sg) % RTgu, T * d.K + j * T, T, all_tokens, 0, 0, 0};
            } else if (t >= t_sd && t < t_ud) {
                const int j = (t - t_sd) / RTd;
                it = Item{IT_DOWN, d.E + j, (t - t_sd) % RTd, T * d.K + j * T, T, 0, 0, 0, 0};
            } else if (routed) {
                const bool gu = t < t_sd;
                const int r = gu ? t - t_ug : t - t_ud;
                const int RT = gu ? RTgu : RTd;
                const int u = r / RT;
                // wait for this expert's plan entry, or for a plan with fewer experts
                unsigned long long v = ld_acquire_u64(entries + u);
                bool skip = false;
                const uint64_t t0 = globaltimer_ns();
                while (!(v >> 63)) {
                    const int f = ld_acquire(&a.ctl[kCtlPlan]);
                    if (f > 0 && u >= f - 1) { skip = true; break; }
                    if (*abort_flag) break;
                    if (globaltimer_ns() - t0 > kWaitNs) { set_error(a, abort_flag, 2); break; }
                    __nanosleep(32);
                    v = ld_acquire_u64(entries + u);
                }
                if (skip) continue;  // fewer distinct experts than the bound
                if (!(v >> 63)) continue;  // aborted
                int toks = 0;
                const int cnt = (int)((v >> 32) & 0xFF);
                for (int i = 0; i < cnt; ++i) toks |= (int)((v >> (40 + 2 * i)) & 3) << (8 * i);
                it = Item{gu ? IT_GU : IT_DOWN, (int)(v & 0xFFFF), r % RT, (int)((v >> 16) & 0xFFFF), cnt, toks, 0, 0, 0};
            }
            if (it.kind == IT_DOWN) it.ready = ld_acquire(&a.ctl[kCtlGuDone + it.ex]) >= RTgu;
        }
        const uint32_t slot = q % kQ;
        if (q >= kQ && !wait_bar(&S.qempty[slot], ((q / kQ) - 1) & 1, abort_flag, a, 3)) it.kind = IT_END;
        if (a.trace) it.pushed_ns = (long long)globaltimer_ns();
        S.items[slot] = it;
        mbar_arrive(&S.qfull[slot]);
        ++q;
        if (it.kind == IT_END) break;
        // A router item's loads (and the plan, when this CTA finishes the last
        // one) would queue behind this SM's in-flight weight copies: start the
        // next item only once the router item is done.
        if (it.kind == IT_ROUTER && !wait_bar(&S.qempty[slot], ((q - 1) / kQ) & 1, abort_flag, a, 12)) continue;
        if (it.kind == IT_GU || it.kind == IT_DOWN) {
            const bool gu = it.kind == IT_GU;
            const int G = gu ? Ggu : Gd;
            const uint8_t* tile = a.weights + (size_t)it.ex * d.expert_stride + (gu ? 0 : d.gu_bytes) +
                                  (size_t)it.rt * G * kBlockBytes;
            const uint32_t stage_bytes = (uint32_t)a.sb * kBlockBytes;
            for (int b0 = 0; b0 < G; b0 += a.sb) {
                const int nb = min(a.sb, G - b0);
                // slot_s = gs % nstages, phase_s = (gs / nstages) & 1
                if (gs >= (uint32_t)a.nstages && !wait_bar(&S.empty[slot_s], phase_s ^ 1, abort_flag, a, 4)) break;
                mbar_arrive_expect_tx(&S.full[slot_s], nb * kBlockBytes);
                bulk_g2s(ring + (size_t)slot_s * stage_bytes, tile + (size_t)b0 * kBlockBytes, nb * kBlockBytes,
                         &S.full[slot_s]);
                ++gs;
                if (++slot_s == (uint32_t)a.nstages) { slot_s = 0; phase_s ^= 1; }
            }
        }
    }
    // let the copies in flight land before the CTA exits (bounded)
    const uint32_t ns = a.nstages;
    for (uint32_t k = (gs > ns ? gs - ns : 0); k < gs; ++k) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&S.full[k % ns], (k / ns) & 1) && globaltimer_ns() - t0 < kWaitNs) {
        }
    }
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Top-k of the T tokens (warp t) and the batch-union plan (all eight warps),
// by the consumers of the CTA that finished the last router item. Each
// distinct expert's packed entry is stored as soon as it is known (a single
// 64-bit store: a producer polling it sees all of it or nothing); the other
// plan arrays are ordered before the one release of the plan flag.
// One token's top-k.
__device__ __forceinline__ void topk_token(const double* l, int E, int K, int lane, int* id, float* wt) {
    if (E <= 256) warp_topk<true, 8>(l, E, K, lane, id, wt);
    else warp_topk<true>(l, E, K, lane, id, wt);
}

__device__ __forceinline__ void consumer_plan(FusedArgs& a, FusedSmem& S, int ctid, int* scnt, int* soff, int* stok) {
    const Dims& d = a.d;
    const int T = a.T, E = d.E, K = d.K, TK = T * K;
    const int cw = ctid >> 5, lane = ctid & 31;
    if (a.trace && ctid == 0) a.trace[4] = (long long)globaltimer_ns();
    if (cw < T) {
        int id;
        float wt;
        topk_token(a.logits + (size_t)cw * E, E, K, lane, &id, &wt);
        if (lane < K) {
            S.sids[cw * K + lane] = id;
            S.sw[cw * K + lane] = wt;
        }
    }
    named_bar(1, kCT);
    if (a.trace && ctid == 0) a.trace[5] = (long long)globaltimer_ns();
    // experts in chunks of 256, 32 per warp: count the slots routed to each,
    // pack their tokens (ascending), scan counts and distinct flags
    unsigned long long* entries = entries_of(a);
    int carry = 0, ucarry = 0;
    for (int c0 = 0; c0 < E; c0 += kCT) {
        const int e = c0 + ctid;
        int c = 0, tk = 0;
        if (e < E) {
            for (int sl = 0; sl < TK; ++sl) {
                if (S.sids[sl] == e) {
                    if (c < 4) tk |= (sl / K) << (8 * c);
                    ++c;
                }
            }
        }
        const int f = c > 0;
        int incl = c, fincl = f;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n1 = __shfl_up_sync(0xffffffffu, incl, o), n2 = __shfl_up_sync(0xffffffffu, fincl, o);
            if (lane >= o) { incl += n1; fincl += n2; }
        }
        if (lane == 31) { S.wsum[cw] = incl; S.wflag[cw] = fincl; }
        named_bar(1, kCT);
        if (a.trace && ctid == 0) a.trace[6] = (long long)globaltimer_ns();
        int base = carry, ubase = ucarry;
        for (int w = 0; w < cw; ++w) { base += S.wsum[w]; ubase += S.wflag[w]; }
        const int off = base + incl - c, rank = ubase + fincl - f;
        if (e < E) {
            if (f) {
                unsigned long long v = (1ull << 63) | (unsigned long long)e | ((unsigned long long)off << 16) |
                                       ((unsigned long long)c << 32);
                for (int i = 0; i < c && i < 4; ++i) v |= (unsigned long long)((tk >> (8 * i)) & 3) << (40 + 2 * i);
                st_relaxed_u64(entries + rank, v);
                a.p.unique[rank] = e;
                a.p.act_expert[rank] = e;
                a.p.act_off[rank] = off;
                a.p.act_cnt[rank] = c;
                a.p.table[rank] = make_int4(e, off, c, tk);
            }
            a.p.off[e] = off;
            a.p.cnt[e] = c;
            soff[e] = off;
        }
        for (int w = 0; w < kCW; ++w) { carry += S.wsum[w]; ucarry += S.wflag[w]; }
        named_bar(1, kCT);
        if (a.trace && ctid == 0) a.trace[7] = (long long)globaltimer_ns();
    }
    const int n_unique = ucarry;
    // slot (t, k): position = first position of its expert + earlier tokens of that expert
    if (ctid < TK) {
        const int e = S.sids[ctid], t = ctid / K;
        int rank = 0;
        for (int sl = 0; sl < t * K; ++sl) rank += S.sids[sl] == e;
        const int q = soff[e] + rank;
        a.p.pos[ctid] = q;
        a.p.tok[q] = t;
        a.p.ids[ctid] = e;
        a.p.w[ctid] = S.sw[ctid];
    }
    for (int i = ctid; i < d.S * T; i += kCT) a.p.tok[TK + i] = i % T;
    for (int j = ctid; j < d.S; j += kCT) {
        a.p.act_expert[n_unique + j] = E + j;
        a.p.act_off[n_unique + j] = TK + j * T;
        a.p.act_cnt[n_unique + j] = T;
    }
    if (ctid == 0) {
        a.p.off[E] = carry;
        *a.p.n_unique = n_unique;
        *a.p.n_active = n_unique + d.S;
    }
    named_bar(1, kCT);
    if (ctid == 0) {
        if (a.trace) a.trace[8] = (long long)globaltimer_ns();
        st_release(&a.ctl[kCtlPlan], n_unique + 1);
        if (a.trace) a.trace[3] = (long long)globaltimer_ns();
    }
}

// ------------------------------------------------------------------ signaler
// y rows of output block rt: residual + shared experts + routed experts in
// routing order (fixed order, same as the separate combine kernel).
template <typename XT>
__device__ void signal_combine(FusedArgs& a, int rt, int lane) {
    const Dims& d = a.d;
    const int T = a.T, K = d.K, TK = T * d.K;
    constexpr int kJ = kTileRows / 32;  // rows per lane: rt * 128 + 32 j + lane
    static_assert(kTileRows % 32 == 0, "a lane covers every 32nd row of the block");
    // every load of a token is issued before its sums (a few round trips per
    // token instead of one per routed slot and row)
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
                    const int q = __shfl_sync(0xffffffffu, q_l, (c0 + c) & 31);
                    const float* orow = a.o + (size_t)q * d.H + rt * kTileRows + lane;
#pragma unroll
                    for (int j = 0; j < kJ; ++j) v[c][j] = c0 + c < nk ? __ldcg(orow + 32 * j) : 0.0f;
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
__device__ void fused_signaler(FusedArgs& a, FusedSmem& S, int lane) {
    const Dims& d = a.d;
    volatile int* abort_flag = &S.abort_flag;
    for (uint32_t k = 0;; ++k) {
        const uint32_t slot = k % kSQ;
        const bool ok = wait_bar(&S.dfull[slot], (k / kSQ) & 1, abort_flag, a, 10);
        const Item r = S.done[slot];
        if (!ok || r.kind == IT_END) break;
        int last = 0;
        if (lane == 0) {
            if (r.kind == IT_GU) {
                red_add_release(&a.ctl[kCtlGuDone + r.ex], 1);
            } else if (r.kind == IT_DOWN) {
                const int prev = atom_add_acq_rel(&a.ctl[kCtlGuDone + d.E + d.S + r.rt], 1);
                // no output block can be complete before the plan is published,
                // so an unpublished plan means this was not the last tile
                const int plan = ld_acquire(&a.ctl[kCtlPlan]);
                last = plan > 0 && prev + 1 == plan - 1 + d.S;
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
// Router rows e0, e0+1: warps 4r..4r+3 take expert e0 + r, each a quarter of
// H, with the weight loads issued before the fp64 products; the four partial
// sums are added in a fixed order.
template <typename XT, int NT>
__device__ void router_item(FusedArgs& a, FusedSmem& S, int e0, int ctid, int* scnt, int* soff, int* stok) {
    const Dims& d = a.d;
    const int cw = ctid >> 5, lane = ctid & 31;
    constexpr int kParts = kCW / kRouterExperts;
    const int r = cw / kParts, part = cw % kParts;
    const int e = e0 + r;
    const int chunk = d.H / kParts;
    const XT* x = reinterpret_cast<const XT*>(a.x);
    double acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[t] = 0.0;
    if (e < d.E) {
        const float* wrow = a.wr + (size_t)e * d.H + part * chunk;
        constexpr int kV = 12;  // float4 per lane per pass: one pass for H = 6144
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
        for (int base = 0; base < chunk; base += kV * 128) {
            // weights and the first token's x in one batch of loads (one round trip)
            float4 wv[kV], xv0[kV];
            const XT* x0 = x + part * chunk;
#pragma unroll
            for (int j = 0; j < kV; ++j) {
                const int i = base + lane * 4 + j * 128;
                wv[j] = i < chunk ? __ldg(reinterpret_cast<const float4*>(wrow + i)) : make_float4(0.f, 0.f, 0.f, 0.f);
                xv0[j] = load_x(x0, i);
            }
            {
                double sacc = 0.0;
#pragma unroll
                for (int j = 0; j < kV; ++j) {
                    sacc = fma((double)wv[j].x, (double)xv0[j].x, sacc);
                    sacc = fma((double)wv[j].y, (double)xv0[j].y, sacc);
                    sacc = fma((double)wv[j].z, (double)xv0[j].z, sacc);
                    sacc = fma((double)wv[j].w, (double)xv0[j].w, sacc);
                }
                acc[0] += sacc;
            }
#pragma unroll 1
            for (int t = 1; t < a.T; ++t) {
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
#pragma unroll
                for (int tt = 1; tt < NT; ++tt)
                    if (tt == t) acc[tt] += sacc;
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
        if (lane == 0) S.rpart[cw][t] = acc[t];
    }
    named_bar(1, kCT);
    if (ctid < kRouterExperts * a.T) {
        const int rr = ctid / a.T, t = ctid % a.T, ee = e0 + rr;
        if (ee < d.E) {
            double sum = 0.0;
            for (int w = 0; w < kParts; ++w) sum += S.rpart[rr * kParts + w][t];
            a.logits[(size_t)t * d.E + ee] = sum + (double)a.bias[ee];
        }
    }
    // the CTA that finishes the last router item builds the plan
    named_bar(1, kCT);
    if (ctid == 0) {
        const int n_router = (d.E + kRouterExperts - 1) / kRouterExperts;
        const uint64_t t0 = a.trace ? globaltimer_ns() : 0;
        S.last = atom_add_acq_rel(&a.ctl[kCtlRouter], 1) == n_router - 1;
        if (S.last && a.trace) { a.trace[1] = (long long)t0; a.trace[2] = (long long)globaltimer_ns(); }
    }
    named_bar(1, kCT);
    if (S.last) consumer_plan(a, S, ctid, scnt, soff, stok);  // uniform: S.last is read after the barrier
}

// Stage the h rows of a down item in B-fragment order, scaled by the powers
// of two that the gate/up items' running maxima select (one pass over h).
__device__ void stage_h(FusedArgs& a, FusedSmem& S, uint4* xb, const Item& it, int ctid, int NT) {
    const int C = a.d.I, G = C / kGroup, L = 8 * NT, nt = it.cnt;
    const unsigned* hm = hmax_of(a);
    if (ctid < nt) {
        const float mx = __uint_as_float(__ldcg(hm + it.off + ctid));
        int k = 0;
        const uint32_t eb = (__float_as_uint(mx) >> 23) & 0xFF;
        if (eb != 0 && eb != 0xFF) {
            k = 14 - ((int)eb - 127);
            k = k < -126 ? -126 : (k > 126 ? 126 : k);
        }
        S.mred[ctid] = exp2i(k);
        S.xscale[ctid] = exp2i(-k);
    }
    named_bar(1, kCT);
    for (int idx = ctid; idx < G * 2 * L; idx += kCT) {
        const int l = idx % L, gh = idx / L;
        const int g = gh >> 1, hh = gh & 1;
        const int n = l >> 2, t = l & 3, j = n >> 1, part = n & 1;
        uint4 o = make_uint4(0u, 0u, 0u, 0u);
        if (j < nt) {
            const float* src = a.h + (size_t)(it.off + j) * C;
            const float f = S.mred[j];
            uint32_t outw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int s = 2 * hh + (q >> 1);
                const int kk = g * 64 + s * 16 + 2 * t + ((q & 1) ? 8 : 0);
                const float2 v = __ldcg(reinterpret_cast<const float2*>(src + kk));
                uint32_t lo;
                const uint32_t hi = split_pair(v.x * f, v.y * f, lo);
                outw[q] = part ? lo : hi;
            }
            o = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        }
        xb[(size_t)gh * L + l] = o;
    }
}

template <typename XT, int NT>
__device__ void weight_item(FusedArgs& a, FusedSmem& S, const Item& it, uint8_t* ring, uint4* xb, float4* corr,
                            uint32_t& slot_s, uint32_t& phase_s, int ctid) {
    const Dims& d = a.d;
    const int cw = ctid >> 5, lane = ctid & 31, gi = lane >> 2, t4 = lane & 3;
    const bool gu = it.kind == IT_GU;
    const int C = gu ? d.H : d.I;
    const int G = C / kGroup;
    const int nt = it.cnt;
    constexpr int L = 8 * NT;  // lanes holding B-fragment columns of NT tokens
    volatile int* abort_flag = &S.abort_flag;

    if (gu) {
        bool same = S.staged_n == nt;
        for (int i = 0; same && i < nt; ++i) same = S.staged_rows[i] == ((it.tokens >> (8 * i)) & 0xFF);
        if (!same) {  // uniform: every consumer reads the same shared values
            int rows[NT];
#pragma unroll
            for (int i = 0; i < NT; ++i) rows[i] = i < nt ? (it.tokens >> (8 * i)) & 0xFF : 0;
            named_bar(1, kCT);  // nobody still reads the previous staging
            stage_bfrag<XT, NT>(xb, S.xscale, reinterpret_cast<const XT*>(a.x), rows, nt, C, false, ctid, kCT, 1,
                                S.mred);
            named_bar(1, kCT);
            stage_offset_corr(xb, corr, G, NT, nt, ctid, kCT);
            named_bar(1, kCT);
            if (ctid == 0) {
                S.staged_n = nt;
                for (int i = 0; i < nt; ++i) S.staged_rows[i] = rows[i];
            }
        }
    } else {
        if (ctid == 0 && !it.ready) wait_geq(&a.ctl[kCtlGuDone + it.ex], 2 * d.I / kTileRows, abort_flag, a, 6);
        named_bar(1, kCT);
        stage_h(a, S, xb, it, ctid, NT);
        named_bar(1, kCT);
        stage_offset_corr(xb, corr, G, NT, nt, ctid, kCT);
        named_bar(1, kCT);
        if (ctid == 0) S.staged_n = -1;
    }

    float acc0 = 0.f, acc1 = 0.f;
    const int sub = cw;
    const uint32_t stage_bytes = (uint32_t)a.sb * kBlockBytes;
    const bool has_b = lane < L;
    const int nst = (G + a.sb - 1) / a.sb;
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
        if (ok) {
            const uint8_t* stage = ring + (size_t)slot_s * stage_bytes;
            const int g0 = i * a.sb;
            const int nb = min(a.sb, G - g0);
#pragma unroll 4
            for (int bb = 0; bb < nb; ++bb) {
                const int g = g0 + bb;
                const uint8_t* bp = stage + bb * kBlockBytes;
                const uint4 w = *reinterpret_cast<const uint4*>(bp + sub * 512 + lane_slot(lane) * 16);
                const uint32_t sv = *reinterpret_cast<const uint32_t*>(bp + kNibbleBytes + sub * 32 + gi * 4);
                uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
                if (has_b) {
                    x0 = xb[(size_t)(g * 2 + 0) * L + lane];
                    x1 = xb[(size_t)(g * 2 + 1) * L + lane];
                }
                group_mma_aw_off(w, sv, x0, x1, corr[g * 4 + t4], acc0, acc1);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.empty[slot_s]);
        if (++slot_s == (uint32_t)a.nstages) { slot_s = 0; phase_s ^= 1; }
        seen = next_full;
    }
    const bool live = t4 < nt && !*abort_flag;
    float hv = 0.0f;
    if (live) {
        const float xs = S.xscale[t4];
        const float v0 = acc0 * xs;  // row gi of the sub-tile
        const float v1 = acc1 * xs;  // row gi+8
        if (gu) {
            // row gi is gate row j, row gi+8 the up row j of the same j
            const int j = (it.rt * 8 + sub) * 8 + gi;
            hv = silu_f(v0) * v1;
            a.h[(size_t)(it.off + t4) * d.I + j] = hv;
        } else {
            const int r0 = it.rt * kTileRows + sub * kSubRows + gi;
            a.o[(size_t)(it.off + t4) * d.H + r0] = v0;
            a.o[(size_t)(it.off + t4) * d.H + r0 + 8] = v1;
        }
    }
    if (gu) {  // running max |h| of each position, for the down items' scaling
        float m = fabsf(hv);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
        if (live && gi == 0) red_max_u32(hmax_of(a) + it.off + t4, __float_as_uint(m));
    }
}

template <typename XT, int NT>
__global__ void __launch_bounds__(kFT, 1) moe_decode_fused_kernel(FusedArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    FusedSmem& S = *reinterpret_cast<FusedSmem*>(smem);
    uint8_t* ring = smem + ((sizeof(FusedSmem) + 127) & ~(size_t)127);
    uint4* xb = reinterpret_cast<uint4*>(ring + (size_t)a.nstages * a.sb * kBlockBytes);
    const int Cmax = a.d.H > a.d.I ? a.d.H : a.d.I;
    float4* corr = reinterpret_cast<float4*>(xb + (size_t)NT * Cmax / 4);  // [Cmax / 64][4] offset corrections
    int* scnt = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(corr) + Cmax);
    int* soff = scnt + a.d.E + 1;
    int* stok = soff + a.d.E + 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < a.nstages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], kCW); }
        for (int i = 0; i < kQ; ++i) { mbar_init(&S.qfull[i], 1); mbar_init(&S.qempty[i], 1); }
        for (int i = 0; i < kSQ; ++i) { mbar_init(&S.dfull[i], kCT); mbar_init(&S.dempty[i], 1); }
        S.abort_flag = 0;
        S.staged_n = -1;
        mbar_fence_init();
        if (a.trace) atomicMin(reinterpret_cast<unsigned long long*>(a.trace) + 9, globaltimer_ns());
    }
    __syncthreads();
    if (warp == kProducerWarp) {
        if (lane == 0) fused_producer(a, S, ring);
        __syncwarp();
    } else if (warp == kSignalWarp) {
        fused_signaler<XT>(a, S, lane);
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
            if (ctid == 0) S.first_wait_ns = S.total_wait_ns = 0;
            if (it.kind == IT_ROUTER) router_item<XT, NT>(a, S, it.ex, ctid, scnt, soff, stok);
            else if (it.kind == IT_GU || it.kind == IT_DOWN)
                weight_item<XT, NT>(a, S, it, ring, xb, corr, slot_s, phase_s, ctid);
            // hand the completion to the signaler: the record first, then every
            // consumer thread arrives after its own global writes
            const uint32_t ds = k % kSQ;
            if (ctid == 0) {
                if (k >= kSQ) wait_bar(&S.dempty[ds], ((k / kSQ) - 1) & 1, &S.abort_flag, a, 11);
                S.done[ds] = it;
            }
            named_bar(1, kCT);
            mbar_arrive(&S.dfull[ds]);
            if (a.trace && ctid == 0 && it.kind != IT_END) {
                const unsigned long long r = atomicAdd(reinterpret_cast<unsigned long long*>(a.trace), 1ull);
                if (r < (unsigned long long)a.trace_cap) {
                    long long* rec = a.trace + 16 + 8 * r;
                    rec[0] = ((long long)blockIdx.x << 40) | ((long long)it.kind << 32) | ((long long)it.ex << 16) | it.rt;
                    rec[1] = (long long)t_begin;
                    rec[2] = (long long)globaltimer_ns();
                    rec[3] = (long long)S.first_wait_ns;
                    rec[4] = it.pushed_ns;
                    rec[5] = (long long)S.total_wait_ns;
                    rec[6] = rec[7] = 0;
                }
            }
            if (ctid == 0 && it.kind != IT_END) mbar_arrive(&S.qempty[slot]);
            ++q;
            if (it.kind == IT_END) break;
        }
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        S.last = atomicAdd(&a.ctl[kCtlExit], 1) == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (S.last) {
        // last CTA out: clear the control block for the next launch (keep the error)
        if (a.trace && tid == 0) a.trace[10] = (long long)globaltimer_ns();
        __threadfence();
        const int n = ctl_ints(a.d.E, a.d.S, a.d.H, a.d.K);
        for (int i = tid; i < n; i += blockDim.x)
            if (i != kCtlError) a.ctl[i] = 0;
        __threadfence();
    }
}

size_t fused_smem_bytes(const Dims& d, int NT, int nstages, int sb) {
    const size_t head = (sizeof(FusedSmem) + 127) & ~(size_t)127;
    const int C = d.H > d.I ? d.H : d.I;
    return head + (size_t)nstages * sb * kBlockBytes + (size_t)NT * C * 4 + (size_t)C + (size_t)(3 * d.E + 3) * 4;
}

// Ring geometry for NT tokens: copies of sb blocks (34,816 B at sb = 8: bulk
// copies that large stream best) and up to max_stages of them in flight per
// SM. More bytes in flight than bandwidth x latency only lengthen the queues
// every dependent load waits in.
static bool fused_geometry(const Dims& d, int NT, size_t smem_limit, int max_stages, int max_sb, int* nstages,
                           int* sb) {
    for (int b = max_sb; b >= 2; b -= 2) {
        int ns = max_stages < kMaxStages ? max_stages : kMaxStages;
        while (ns > 0 && fused_smem_bytes(d, NT, ns, b) > smem_limit) --ns;
        if (ns >= 2) { *nstages = ns; *sb = b; return true; }
    }
    return false;
}

int fused_stages_for(const Dims& d, int NT, size_t smem_limit) {
    int ns = 0, sb = 0;
    return fused_geometry(d, NT, smem_limit, kMaxStages, kMaxSB, &ns, &sb) ? ns : 0;
}

template <typename XT, int NT>
static cudaError_t launch_fused_t(const FusedArgs& a, int n_sm, size_t smem_limit, cudaStream_t st) {
    static int configured_device = -1;  // the opt-in limit is set once per device
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(moe_decode_fused_kernel<XT, NT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_limit);
        if (e != cudaSuccess) return e;
        configured_device = dev;
    }
    const size_t smem = fused_smem_bytes(a.d, NT, a.nstages, a.sb);
    moe_decode_fused_kernel<XT, NT><<<n_sm, kFT, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_decode_fused(const uint8_t* weights, const Dims& d, const float* wr, const float* bias,
                                const void* x, coli_dtype dt, int T, void* y, const float* residual, const Plan& p,
                                double* logits, float* h, float* o, int* ctl, int n_sm, size_t smem_limit,
                                long long* trace, int trace_cap, int max_stages, int max_sb, cudaStream_t st) {
    if (T < 1 || T > kFusedMaxTok) return cudaErrorInvalidValue;
    const int NT = T == 1 ? 1 : (T == 2 ? 2 : 4);
    FusedArgs a;
    a.weights = weights; a.d = d; a.wr = wr; a.bias = bias; a.x = x; a.y = y; a.residual = residual;
    a.T = T; a.p = p; a.logits = logits; a.h = h; a.o = o; a.ctl = ctl;
    a.trace = trace; a.trace_cap = trace_cap;
    a.umax = T * d.K < d.E ? T * d.K : d.E;
    if (!fused_geometry(d, NT, smem_limit, max_stages, max_sb, &a.nstages, &a.sb))
        return cudaErrorInvalidConfiguration;
    if (dt == COLI_F32) {
        if (NT == 1) return launch_fused_t<float, 1>(a, n_sm, smem_limit, st);
        if (NT == 2) return launch_fused_t<float, 2>(a, n_sm, smem_limit, st);
        return launch_fused_t<float, 4>(a, n_sm, smem_limit, st);
    }
    if (NT == 1) return launch_fused_t<__nv_bfloat16, 1>(a, n_sm, smem_limit, st);
    if (NT == 2) return launch_fused_t<__nv_bfloat16, 2>(a, n_sm, smem_limit, st);
    return launch_fused_t<__nv_bfloat16, 4>(a, n_sm, smem_limit, st);
}

}  // namespace coli
