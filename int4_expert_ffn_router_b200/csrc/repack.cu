// repack.cu -- canonical int4 gs64 container -> device-native tile layout
// (described in common.cuh). Runs once per expert at layer creation.
#include "common.cuh"
#include "kernels.cuh"

namespace coli {

// One thread per output 32-bit word (8 nibbles). For the interleaved
// gate/up matrix, combined row 16b+i is gate row 8b+i (i < 8) or up row
// 8b+i-8 (i >= 8).
__global__ void repack_kernel(const uint8_t* __restrict__ q0, const uint16_t* __restrict__ s0,
                              const uint8_t* __restrict__ q1, const uint16_t* __restrict__ s1, int R, int C,
                              int interleave_gu, uint8_t* __restrict__ dst) {
    const int G = C / kGroup;
    const long long total = (long long)R * C / 8;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int s = (int)(idx & 3);
        const int lane = (int)((idx >> 2) & 31);
        const int sub = (int)((idx >> 7) & 7);
        const long long blk = idx >> 10;  // rt * G + g
        const int g = (int)(blk % G);
        const int rt = (int)(blk / G);
        const int gi = lane >> 2, ti = lane & 3;
        const int ra = rt * kTileRows + sub * kSubRows + gi;  // combined row of nibble rows "gi"
        const uint8_t *rowa, *rowb;
        const uint16_t *sca, *scb;
        if (interleave_gu) {
            const int src = (ra >> 4) * 8 + (ra & 7);  // same index in gate (row a) and up (row b)
            rowa = q0 + (size_t)src * (C / 2);
            rowb = q1 + (size_t)src * (C / 2);
            sca = s0 + (size_t)src * G;
            scb = s1 + (size_t)src * G;
        } else {
            rowa = q0 + (size_t)ra * (C / 2);
            rowb = q0 + (size_t)(ra + 8) * (C / 2);
            sca = s0 + (size_t)ra * G;
            scb = s0 + (size_t)(ra + 8) * G;
        }
        const int cb0 = g * 32 + s * 8 + ti, cb1 = cb0 + 4;
        const uint32_t b00 = rowa[cb0], b01 = rowa[cb1], b10 = rowb[cb0], b11 = rowb[cb1];
        uint32_t w = (b00 & 0xF) | ((b10 & 0xF) << 4) | ((b01 & 0xF) << 8) | ((b11 & 0xF) << 12) |
                     ((b00 >> 4) << 16) | ((b10 >> 4) << 20) | ((b01 >> 4) << 24) | ((b11 >> 4) << 28);
        w ^= 0x88888888u;  // two's complement code q -> offset binary q + 8
        uint8_t* block = dst + (size_t)blk * kBlockBytes;
        reinterpret_cast<uint32_t*>(block + sub * 512 + lane_slot(lane) * 16)[s] = w;
        if (ti == 0 && s == 0) {
            const uint32_t pair = (uint32_t)sca[g] | ((uint32_t)scb[g] << 16);
            reinterpret_cast<uint32_t*>(block + kNibbleBytes + sub * 32)[gi] = pair;
        }
    }
}

cudaError_t launch_repack(const uint8_t* q0, const uint16_t* s0, const uint8_t* q1, const uint16_t* s1, int R, int C,
                          bool interleave_gu, uint8_t* dst, cudaStream_t st) {
    long long total = (long long)R * C / 8;
    long long grid = (total + 255) / 256;
    if (grid > 148LL * 32) grid = 148LL * 32;
    repack_kernel<<<(int)grid, 256, 0, st>>>(q0, s0, q1, s1, R, C, interleave_gu ? 1 : 0, dst);
    return cudaGetLastError();
}

}  // namespace coli
