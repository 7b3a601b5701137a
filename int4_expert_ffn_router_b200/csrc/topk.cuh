// topk.cuh -- warp-level top-k selection with softmax renormalisation.
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kMaxPerLane = 32;  // E <= 1024

// Order-preserving 64-bit key of a double (larger value -> larger key); -0 is
// folded into +0 so that equal values compare equal. Integer compares keep
// the selection exact and are much cheaper than fp64 ones.
__device__ __forceinline__ unsigned long long order_key(double v) {
    unsigned long long u = (unsigned long long)__double_as_longlong(v + 0.0);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// One warp selects the K largest of the E logits l[0..E) (descending, ties to
// the lower id) and their softmax weights over the selection (fp64, fixed
// summation order). Lane k < K returns slot k in (*id, *wt). Each lane keeps
// the best of its own values; a round takes the warp's best (three warp
// reductions: the key's high word, its low word among the lanes holding that
// high word, the lowest id among the lanes holding the key) and only the lane
// that supplied it refreshes its own best. `coherent`: read the logits
// through L2 only (they were written by another CTA).
// Inverse of order_key.
__device__ __forceinline__ double key_value(unsigned long long k) {
    const unsigned long long u = (k >> 63) ? (k & 0x7FFFFFFFFFFFFFFFull) : ~k;
    return __longlong_as_double((long long)u);
}

// Weights of the selection (lane k < K holds slot k: its key, its id) and
// the adaptive expert top-p ("colibri: 1300 lines of C ..." (jsqmd.com),
// usage section: topp, adaptive expert top-p). w_k = exp(l_k - l_0) / z over
// the K selected logits (fp64). With 0 < topp < 1 the slots are kept while
// the running sum of w in slot order (fp64, sequential) has not yet reached
// topp, the first slot that reaches it included; the kept weights are
// divided by that sum, and each dropped slot repeats slot 0's id with weight
// 0, so the batch-union gains nothing from it and the combine adds exactly 0.
__device__ __forceinline__ void topk_weights(unsigned long long my_key, unsigned long long top_key, int my_id, int K,
                                             double topp, int lane, int* id_out, float* wt_out) {
    const double ex = (lane < K) ? exp(key_value(my_key) - key_value(top_key)) : 0.0;
    double z = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const double w = ex / z;
    if (!(topp > 0.0 && topp < 1.0)) {
        *id_out = my_id;
        *wt_out = (float)w;
        return;
    }
    int keep = K;
    double cum = 0.0, cum_keep = 0.0;
    for (int j = 0; j < K; ++j) {
        cum += __shfl_sync(0xffffffffu, w, j);
        if (keep == K && cum >= topp) {
            keep = j + 1;
            cum_keep = cum;
        }
    }
    if (keep == K) cum_keep = cum;
    const int first = __shfl_sync(0xffffffffu, my_id, 0);
    *id_out = lane < keep ? my_id : first;
    *wt_out = lane < keep ? (float)(w / cum_keep) : 0.0f;
}

template <bool coherent, int PER = kMaxPerLane>
__device__ __forceinline__ void warp_topk(const double* __restrict__ l, int E, int K, double topp, int lane, int* id,
                                          float* wt) {
    const int per = (E + 31) / 32;  // <= PER
    unsigned long long key[PER];     // 0: absent or taken (below every logit's key)
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        key[i] = 0ull;
        if (i < per && e < E) key[i] = order_key(coherent ? __ldcg(l + e) : l[e]);
    }
    // this lane's best: largest key, then lowest id (lower i = lower id)
    unsigned long long mk = 0ull;
    int mi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        if (key[i] > mk) { mk = key[i]; mi = lane + 32 * i; }
    }
    unsigned long long my_key = 0ull, top_key = 0ull;
    int my_id = -1;
    for (int k = 0; k < K; ++k) {
        // the warp's best: largest key (high word, then low word), then lowest id
        const unsigned khi = (unsigned)(mk >> 32), klo = (unsigned)mk;
        const unsigned bhi = __reduce_max_sync(0xffffffffu, khi);
        const unsigned blo = __reduce_max_sync(0xffffffffu, khi == bhi ? klo : 0u);
        const bool holds = khi == bhi && klo == blo;
        const int bi = (int)__reduce_min_sync(0xffffffffu, holds ? (unsigned)mi : 0x7fffffffu);
        const unsigned long long bk = ((unsigned long long)bhi << 32) | blo;
        if ((bi & 31) == lane && bi != 0x7fffffff) {  // the supplier drops it and refreshes its best
            mk = 0ull;
            mi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                if (lane + 32 * i == bi) key[i] = 0ull;
                if (key[i] > mk) { mk = key[i]; mi = lane + 32 * i; }
            }
        }
        if (k == 0) top_key = bk;
        if (lane == k) { my_key = bk; my_id = bi; }
    }
    topk_weights(my_key, top_key, my_id, K, topp, lane, id, wt);
}

// The same selection for E <= 256 (at most 8 logits per lane), faster: each
// lane first sorts its own keys (descending key, then ascending id) with a
// fixed 19-comparator network, so a round only compares the lanes' heads
// (three warp reductions) and the supplier shifts its list by one.
// Identical results to warp_topk.
__device__ __forceinline__ void cx8(unsigned long long (&k)[8], int (&id)[8], int a, int b) {
    // after the exchange, slot a holds the entry that comes first
    const bool swap = k[b] > k[a] || (k[b] == k[a] && id[b] < id[a]);
    const unsigned long long ka = swap ? k[b] : k[a], kb = swap ? k[a] : k[b];
    const int ia = swap ? id[b] : id[a], ib = swap ? id[a] : id[b];
    k[a] = ka; k[b] = kb; id[a] = ia; id[b] = ib;
}

template <bool coherent>
__device__ __forceinline__ void warp_topk8(const double* __restrict__ l, int E, int K, double topp, int lane,
                                           int* id_out, float* wt_out) {
    unsigned long long k[8];
    int id[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        k[i] = 0ull;
        id[i] = 0x7fffffff;
        if (e < E) {
            k[i] = order_key(coherent ? __ldcg(l + e) : l[e]);
            id[i] = e;
        }
    }
    // Batcher's odd-even merge sort of 8 entries (19 comparators)
    cx8(k, id, 0, 1); cx8(k, id, 2, 3); cx8(k, id, 4, 5); cx8(k, id, 6, 7);
    cx8(k, id, 0, 2); cx8(k, id, 1, 3); cx8(k, id, 4, 6); cx8(k, id, 5, 7);
    cx8(k, id, 1, 2); cx8(k, id, 5, 6);
    cx8(k, id, 0, 4); cx8(k, id, 1, 5); cx8(k, id, 2, 6); cx8(k, id, 3, 7);
    cx8(k, id, 2, 4); cx8(k, id, 3, 5);
    cx8(k, id, 1, 2); cx8(k, id, 3, 4); cx8(k, id, 5, 6);
    unsigned long long my_key = 0ull, top_key = 0ull;
    int my_id = -1;
    for (int r = 0; r < K; ++r) {
        const unsigned khi = (unsigned)(k[0] >> 32), klo = (unsigned)k[0];
        const unsigned bhi = __reduce_max_sync(0xffffffffu, khi);
        const unsigned blo = __reduce_max_sync(0xffffffffu, khi == bhi ? klo : 0u);
        const bool holds = khi == bhi && klo == blo;
        const int bi = (int)__reduce_min_sync(0xffffffffu, holds ? (unsigned)id[0] : 0x7fffffffu);
        const unsigned long long bk = ((unsigned long long)bhi << 32) | blo;
        if (holds && id[0] == bi) {  // the supplier drops its head
#pragma unroll
            for (int i = 0; i < 7; ++i) { k[i] = k[i + 1]; id[i] = id[i + 1]; }
            k[7] = 0ull;
            id[7] = 0x7fffffff;
        }
        if (r == 0) top_key = bk;
        if (lane == r) { my_key = bk; my_id = bi; }
    }
    topk_weights(my_key, top_key, my_id, K, topp, lane, id_out, wt_out);
}

}  // namespace coli
