// topk.cuh -- warp-level top-k selection with softmax renormalisation.
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kMaxPerLane = 32;  // E <= 1024

__device__ __forceinline__ bool better(double a, int ia, double b, int ib) {
    return a > b || (a == b && ia < ib);
}

// Order-preserving 64-bit key of a double (larger value -> larger key); -0 is
// folded into +0 so that equal values compare equal. Integer compares keep
// the selection exact and are much cheaper than fp64 ones.
__device__ __forceinline__ unsigned long long order_key(double v) {
    unsigned long long u = (unsigned long long)__double_as_longlong(v + 0.0);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

__device__ __forceinline__ bool key_better(unsigned long long ka, int ia, unsigned long long kb, int ib) {
    return ka > kb || (ka == kb && ia < ib);
}

// One warp selects the K largest of the E logits l[0..E) (descending, ties to
// the lower id) and their softmax weights over the selection (fp64, fixed
// summation order). Lane k < K returns slot k in (*id, *wt). Each lane keeps
// the best of its own values; a round takes the warp's best and only the lane
// that supplied it refreshes its own best. `coherent`: read the logits
// through L2 only (they were written by another CTA).
template <bool coherent, int PER = kMaxPerLane>
__device__ __forceinline__ void warp_topk(const double* __restrict__ l, int E, int K, int lane, int* id, float* wt) {
    const int per = (E + 31) / 32;  // <= PER
    double v[PER];
    unsigned long long key[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        int e = lane + 32 * i;
        double val = -INFINITY;
        if (i < per && e < E) val = coherent ? __ldcg(l + e) : l[e];
        v[i] = val;
        key[i] = (i < per && e < E) ? order_key(val) : 0ull;  // key 0: below every logit
    }
    // this lane's best: largest key, then lowest id (lower i = lower id)
    auto local_best = [&](unsigned long long& bk, int& bi) {
        bk = 0ull;
        bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int e = lane + 32 * i;
            if (i < per && e < E && key_better(key[i], e, bk, bi)) { bk = key[i]; bi = e; }
        }
    };
    unsigned long long mk;
    int mi;
    local_best(mk, mi);
    double my_sel = 0.0, top = 0.0;
    int my_id = -1;
    for (int k = 0; k < K; ++k) {
        unsigned long long bk = mk;
        int bi = mi;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const unsigned long long ok = __shfl_xor_sync(0xffffffffu, bk, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (key_better(ok, oi, bk, bi)) { bk = ok; bi = oi; }
        }
        const bool mine = (bi & 31) == lane && bi != 0x7fffffff;
        double bv = 0.0;
        if (mine) {
#pragma unroll
            for (int i = 0; i < PER; ++i)
                if (lane + 32 * i == bi) { bv = v[i]; key[i] = 0ull; }  // taken
            local_best(mk, mi);
        }
        bv = __shfl_sync(0xffffffffu, bv, bi & 31);
        if (k == 0) top = bv;
        if (lane == k) { my_sel = bv; my_id = bi; }
    }
    double ex = (lane < K) ? exp(my_sel - top) : 0.0;
    double z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    *id = my_id;
    *wt = (float)(ex / z);
}

}  // namespace coli
