// clock_stamp.cu -- a measurement aid: per-SM clock and global-timer stamps.
//
// Two stamps taken around a timed region give each SM's mean clock rate over
// that region (SM clock cycles elapsed / nanoseconds elapsed), which a
// sampling tool cannot see in regions of a few milliseconds.
#include <string>

#include "common.cuh"
#include "kernels.cuh"

#define COLI_API extern "C" __attribute__((visibility("default")))

namespace {

// Block b writes {SM id, SM clock (clock64), global timer (ns)} at 3 b.
__global__ void clock_stamp_kernel(long long* out) {
    if (threadIdx.x != 0) return;
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    long long c;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
    const long long t = (long long)coli::globaltimer_ns();
    out[3 * blockIdx.x] = smid;
    out[3 * blockIdx.x + 1] = c;
    out[3 * blockIdx.x + 2] = t;
}

}  // namespace

COLI_API coli_status coli_clock_stamp(long long* buffer, int n_blocks, coli_stream stream) {
    if (!buffer || n_blocks < 1 || n_blocks > 65535) {
        coli::set_last_error("buffer is NULL or n_blocks out of [1, 65535]");
        return COLI_EINVAL;
    }
    clock_stamp_kernel<<<n_blocks, 32, 0, (cudaStream_t)stream>>>(buffer);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        coli::set_last_error(std::string("clock stamp: ") + cudaGetErrorString(e));
        return COLI_ECUDA;
    }
    return COLI_OK;
}
