// route_noalloc.cu -- routing (router logits, top-k, renormalised weights)
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they route tokens:
// code running while a stream is being captured into a CUDA graph (allocation
// calls are not allowed there), code that owns a fixed memory budget handed
// out by another framework's pool, and code on paths that must not block on
// the driver's allocator. coli_moe_route needs a layer, whose workspace is
// allocated at create time; this entry point needs neither: its only scratch,
// the fp64 logits, lives in a fixed array in device memory that every GPU
// loading the library holds until the process exits.
#include <cuda.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "kernels.cuh"

#define COLI_API extern "C" __attribute__((visibility("default")))

namespace {

// fp64 logits of up to COLI_NOALLOC_MAX_TOKENS x COLI_NOALLOC_MAX_EXPERTS
// (504 KiB). Every call on a device shares it and it keeps the last call's
// values; the router kernel writes every logit it later reads, so nothing in
// it has to start at zero. The token limit stays below the batch size from
// which coli_moe_route switches to its split blocked form, so both entry
// points sum every logit in the same order.
static_assert(COLI_NOALLOC_MAX_TOKENS < coli::kRouterGemmMinTok,
              "the no-alloc routing must sum logits in the same order as coli_moe_route");
__device__ __align__(256) double g_noalloc_logits[COLI_NOALLOC_MAX_TOKENS * COLI_NOALLOC_MAX_EXPERTS];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
// Device address of g_noalloc_logits per device, with the id of the context
// it was looked up in: a device reset makes a new context (new id) in which
// the module, and the array, may sit at another address.
double* g_scratch[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Id of the calling thread's current context, or 0 when it cannot be read
// (then the address is looked up on every call).
unsigned long long current_ctx_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool resolved = false;
    if (!resolved) {
        void* f0 = nullptr;
        void* f1 = nullptr;
        cudaDriverEntryPointQueryResult q0, q1;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f0, cudaEnableDefault, &q0) == cudaSuccess &&
            q0 == cudaDriverEntryPointSuccess &&
            cudaGetDriverEntryPoint("cuCtxGetId", &f1, cudaEnableDefault, &q1) == cudaSuccess &&
            q1 == cudaDriverEntryPointSuccess) {
            get_current = reinterpret_cast<CtxGetCurrentFn>(f0);
            get_id = reinterpret_cast<CtxGetIdFn>(f1);
        }
        resolved = true;
    }
    if (!get_current || !get_id) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

coli_status fail(coli_status s, const std::string& what) {
    coli::set_last_error(what);  // reported by coli_last_error()
    return s;
}

}  // namespace

COLI_API coli_status coli_moe_route_noalloc(const float* router_w, const float* router_bias, int n_experts, int hidden,
                                            int top_k, const void* x, coli_dtype dtype, int n_tokens, int32_t* ids,
                                            float* weights, coli_stream stream) {
    if (n_tokens < 0 || n_tokens > COLI_NOALLOC_MAX_TOKENS)
        return fail(COLI_EINVAL, "n_tokens must be in [0, " + std::to_string(COLI_NOALLOC_MAX_TOKENS) +
                                     "] (the fixed scratch holds that many tokens)");
    if (n_experts < 1 || n_experts > COLI_NOALLOC_MAX_EXPERTS)
        return fail(COLI_EINVAL, "n_experts must be in [1, " + std::to_string(COLI_NOALLOC_MAX_EXPERTS) + "]");
    if (top_k < 1 || top_k > n_experts || top_k > 32) return fail(COLI_EINVAL, "top_k must be in [1, min(n_experts, 32)]");
    if (hidden <= 0 || hidden % 128) return fail(COLI_EINVAL, "hidden must be a positive multiple of 128");
    if (dtype != COLI_F32 && dtype != COLI_BF16) return fail(COLI_EINVAL, "dtype must be COLI_F32 or COLI_BF16");
    if (n_tokens == 0) return COLI_OK;
    if (!router_w || !x || !ids || !weights) return fail(COLI_EINVAL, "NULL pointer argument");
    if (((uintptr_t)router_w | (uintptr_t)x) & 15u) return fail(COLI_EINVAL, "router_w and x must be 16-byte aligned");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(COLI_ECUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(COLI_EUNSUPPORTED, "device index above 63");
    double* scratch = nullptr;
    {
        // First call on a device (or in a new context after a device reset):
        // look up the device address of the array, with that device current
        // (in host code its name is only a host-side stand-in).
        std::lock_guard<std::mutex> lock(g_mutex);
        const unsigned long long ctx = g_scratch[dev] ? current_ctx_id() : 0;
        if (!g_scratch[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_noalloc_logits);
            if (e != cudaSuccess) return fail(COLI_ECUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
            g_scratch[dev] = static_cast<double*>(p);
            g_scratch_ctx[dev] = current_ctx_id();
        }
        scratch = g_scratch[dev];
    }
    cudaStream_t s = (cudaStream_t)stream;
    e = coli::launch_router_logits(router_w, router_bias, x, dtype, n_tokens, hidden, n_experts, scratch, s);
    if (e != cudaSuccess) return fail(COLI_ECUDA, std::string("router: ") + cudaGetErrorString(e));
    e = coli::launch_topk(scratch, n_tokens, n_experts, top_k, ids, weights, s);
    if (e != cudaSuccess) return fail(COLI_ECUDA, std::string("topk: ") + cudaGetErrorString(e));
    return COLI_OK;
}
