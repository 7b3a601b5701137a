/*
 * synth_dev.cu -- device twin of the seeded synthetic input generator
 * (definitions in synth_core.h, shared with synth_host.c). It writes the same
 * canonical bytes as the host generator straight into device memory, so a
 * 5 GB layer is built in milliseconds instead of minutes on the host. Test and
 * benchmark infrastructure only; it computes nothing of the MoE layer.
 */
#include <cuda_runtime.h>
#include "synth_core.h"

#define SYNTH_API extern "C" __attribute__((visibility("default")))

/* One thread per 64-element group of `n_experts` consecutive experts. */
__global__ void synth_expert_kernel(uint64_t seed, int layer, int expert0, int n_experts, int H, int I,
                                    float wscale, uint8_t* q, uint16_t* s)
{
    const long long gpm_gu = (long long)I * (H / 64);    /* groups of gate (and of up) */
    const long long gpm_d = (long long)H * (I / 64);     /* groups of down             */
    const long long per_expert = 2 * gpm_gu + gpm_d;
    const long long total = per_expert * n_experts;
    for (long long gid = blockIdx.x * (long long)blockDim.x + threadIdx.x; gid < total;
         gid += (long long)gridDim.x * blockDim.x) {
        int ei = (int)(gid / per_expert);
        long long w = gid - (long long)ei * per_expert;
        int matrix, cols, r, g;
        long long sbase;
        if (w < gpm_gu) { matrix = SYNTH_M_GATE; cols = H; sbase = 0; }
        else if (w < 2 * gpm_gu) { matrix = SYNTH_M_UP; cols = H; w -= gpm_gu; sbase = gpm_gu; }
        else { matrix = SYNTH_M_DOWN; cols = I; w -= 2 * gpm_gu; sbase = 2 * gpm_gu; }
        int groups = cols / 64;
        r = (int)(w / groups);
        g = (int)(w - (long long)r * groups);
        uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_EXPERT, (uint32_t)(expert0 + ei), (uint32_t)matrix);
        __align__(16) uint8_t bytes[32];
        uint16_t sc;
        synth_weight_group(key, cols, r, g, wscale, bytes, &sc);
        long long sidx = (long long)ei * per_expert + sbase + (long long)r * groups + g;
        s[sidx] = sc;
        uint4* dst = reinterpret_cast<uint4*>(q + sidx * 32);
        const uint4* src = reinterpret_cast<const uint4*>(bytes);
        dst[0] = src[0];
        dst[1] = src[1];
    }
}

__global__ void synth_router_kernel(uint64_t seed, int layer, int E, int H, float wscale, float* wr)
{
    uint64_t key = synth_key(seed, (uint32_t)layer, SYNTH_T_ROUTER, 0, 0);
    long long n = (long long)E * H;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        wr[i] = SYNTH_MUL(wscale, synth_gauss(key, (uint64_t)i));
}

__global__ void synth_x_kernel(uint64_t seed, int step, long long n, float* xf, uint16_t* xb)
{
    uint64_t key = synth_key(seed, 0, SYNTH_T_X, (uint32_t)step, 0);
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        float z = synth_gauss(key, (uint64_t)i);
        if (xf) xf[i] = z;
        else xb[i] = synth_f32_to_bf16(z);
    }
}

static int grid_for(long long n, int block)
{
    long long g = (n + block - 1) / block;
    if (g > 148LL * 64) g = 148LL * 64;
    return (int)(g < 1 ? 1 : g);
}

/* q and s must hold n_experts canonical experts (16-byte aligned q). Returns a cudaError_t. */
SYNTH_API int synth_expert_dev(uint64_t seed, int layer, int expert0, int n_experts, int H, int I,
                               float wscale, void* q, void* s, void* stream)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64 || n_experts <= 0 || !q || !s) return (int)cudaErrorInvalidValue;
    if (((uintptr_t)q) & 15u) return (int)cudaErrorInvalidValue;
    long long total = (3LL * H * I / 64) * n_experts;
    synth_expert_kernel<<<grid_for(total, 128), 128, 0, (cudaStream_t)stream>>>(
        seed, layer, expert0, n_experts, H, I, wscale, (uint8_t*)q, (uint16_t*)s);
    return (int)cudaGetLastError();
}

SYNTH_API int synth_router_dev(uint64_t seed, int layer, int E, int H, float wscale, void* wr, void* stream)
{
    if (E <= 0 || H <= 0 || !wr) return (int)cudaErrorInvalidValue;
    long long n = (long long)E * H;
    synth_router_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(seed, layer, E, H, wscale, (float*)wr);
    return (int)cudaGetLastError();
}

/* dtype 0: fp32 output, 1: bf16 bits. */
SYNTH_API int synth_x_dev(uint64_t seed, int step, int T, int H, int dtype, void* x, void* stream)
{
    if (T < 0 || H <= 0 || (T && !x) || (dtype != 0 && dtype != 1)) return (int)cudaErrorInvalidValue;
    if (T == 0) return 0;
    long long n = (long long)T * H;
    synth_x_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(
        seed, step, n, dtype == 0 ? (float*)x : nullptr, dtype == 1 ? (uint16_t*)x : nullptr);
    return (int)cudaGetLastError();
}
