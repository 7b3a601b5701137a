// topk.cuh -- warp-level top-k selection with softmax renormalisation.
#pragma once

#include "common.cuh"

namespace coli {

constexpr int kMaxPerLane = 32;  // E <= 1024

__device__ __forceinline__ bool better(double a, int ia, double b, int ib) {
    return a > b || (a == b && ia < ib);
}

// One warp selects the K largest of the E logits l[0..E) (descending, ties to
// the lower id) and their softmax weights over the selection (fp64, fixed
// summation order). Lane k < K returns slot k in (*id, *wt). `coherent`:
// read the logits through L2 only (they were written by another CTA).
template <bool coherent, int PER = kMaxPerLane>
__device__ __forceinline__ void warp_topk(const double* __restrict__ l, int E, int K, int lane, int* id, float* wt) {
    const int per = (E + 31) / 32;  // <= PER
    double v[PER];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        int e = lane + 32 * i;
        double val = -INFINITY;
        if (i < per && e < E) val = coherent ? __ldcg(l + e) : l[e];
        v[i] = val;
    }
    double my_sel = 0.0, top = 0.0;
    int my_id = -1;
    for (int k = 0; k < K; ++k) {
        double bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            int e = lane + 32 * i;
            if (i < per && e < E && !((taken >> i) & 1u) && better(v[i], e, bv, bi)) { bv = v[i]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
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
