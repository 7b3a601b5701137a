// layer.cu -- the C ABI (include/coli_moe.h): layer object, weight upload and
// repack, workspace, and the forward sequence on one stream.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "expert_cache.h"
#include "kernels.cuh"

#define COLI_API extern "C" __attribute__((visibility("default")))

using namespace coli;

namespace {
thread_local std::string g_last_error;

coli_status fail(coli_status s, const char* what) {
    g_last_error = what;
    return s;
}

coli_status cuda_fail(cudaError_t e, const char* where) {
    g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
    return COLI_ECUDA;
}

#define CUDA_TRY(call, where)                         \
    do {                                              \
        cudaError_t _e = (call);                      \
        if (_e != cudaSuccess) return cuda_fail(_e, where); \
    } while (0)

size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }

// Testing aid (coli_moe_debug_fail_alloc): when positive, the allocation
// that brings the count to zero fails as if the device were out of memory.
std::atomic<int> g_fail_alloc{0};

bool planned_failure() {
    int k = g_fail_alloc.load();
    while (k > 0 && !g_fail_alloc.compare_exchange_weak(k, k - 1)) {
    }
    return k == 1;
}

// Every device allocation of a layer goes through here.
cudaError_t dev_alloc(void** p, size_t bytes) {
    *p = nullptr;
    if (planned_failure()) return cudaErrorMemoryAllocation;
    return cudaMalloc(p, bytes);
}

// And every page-locked host allocation (the expert cache's backing store).
template <typename T>
cudaError_t host_alloc(T** p, size_t bytes) {
    *p = nullptr;
    if (planned_failure()) return cudaErrorMemoryAllocation;
    void* v = nullptr;
    cudaError_t e = cudaHostAlloc(&v, bytes, cudaHostAllocDefault);
    *p = static_cast<T*>(v);
    return e;
}

template <typename T>
cudaError_t dev_alloc(T** p, size_t bytes) {
    void* v = nullptr;
    cudaError_t e = dev_alloc(&v, bytes);
    *p = static_cast<T*>(v);
    return e;
}

// Switches to `dev` for the lifetime of the guard.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) prev = -1;
        if (prev != dev) ok = cudaSetDevice(dev) == cudaSuccess;
    }
    ~DeviceGuard() {
        int cur = -1;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}
}  // namespace

struct coli_moe_layer {
    coli_moe_config cfg;
    Dims d;
    int device = 0;
    int n_sm = 148;
    int max_active = 0;
    uint8_t* weights = nullptr;
    float* router_w = nullptr;
    float* router_b = nullptr;
    uint8_t* ws = nullptr;
    size_t ws_bytes = 0;
    double* logits = nullptr;
    int64_t launches = 0;  // kernels of this library enqueued by route/forward/stack calls
    Plan plan{};
    float* h = nullptr;
    float* o = nullptr;
    float* xn = nullptr;
    int* ctl = nullptr;             // control block of the persistent decode kernels
    int ctl_n = 0;                  // its ints
    // integer-MMA persistent kernel (decode_i8.cu): token parts and SwiGLU output parts
    uint8_t* xq = nullptr;
    uint8_t* xm = nullptr;
    uint8_t* hq = nullptr;
    uint8_t* hm = nullptr;
    int i8_max_tok = 0;             // largest batch its workspace holds
    int64_t wait_ns = 0;            // bound of its waits (0: 1 s)
    int wait_test = 0;              // testing aid (coli_moe_debug_wait_test)
    // tensor-core path (bf16 batches too large for the persistent kernel)
    __half* xs = nullptr;           // [2 slots][H] scaled fp16 rows of x in position order (hi, lo for fp32 x)
    float4* tscale = nullptr;       // [max_tokens] per-token power-of-two scales
    float4* slot = nullptr;         // [slots] per-position epilogue factors
    int4* tiles = nullptr;          // tile list
    int* n_tiles = nullptr;
    unsigned* meta = nullptr;       // [0] max L1(gate row) * L1(up row), [1] max |scale| (float bits)
    double* rpart = nullptr;        // router partial sums (split input dimension)
    // certified integer-MMA router of token batches (router_certified.cu)
    bool cert_ok = false;           // shapes and device allow it and the workspace holds its buffers
    RouterCert rc;
    alignas(64) unsigned char rc_maps[6 * kTensorMapBytes] = {};  // TMA maps of its digit planes
    size_t rpart_cap = 0;           // doubles
    bool tc_shape_ok = false;       // shapes and shared memory allow the tensor-core kernels
    bool tc_scale_ok = true;        // every weight scale keeps q * scale finite in fp16
    int tc_mode = 1;                // coli_moe_set_tensor_cores: 0 CUDA cores, 1 bf16 on tensor cores, 2 bf16 and fp32
    alignas(64) unsigned char xs_maps[2 * kTensorMapBytes] = {};  // TMA maps of the token operands
    alignas(64) unsigned char h16_maps[2 * kTensorMapBytes] = {};  // (boxes of kTcMaxTok and 32 rows)
    size_t smem_optin = 0;
    int fused = 1;                  // coli_moe_set_fused: 1 persistent kernel for small batches, 0 separate kernels
    double topp = 1.0;              // coli_moe_set_expert_top_p (1: plain top-K)
    long long* trace = nullptr;     // caller-owned device buffer for the item timeline
    int trace_cap = 0;
    int ring_stages = kDefaultStages;        // persistent kernel: bulk copies in flight per SM
    int ring_blocks = kDefaultStageBlocks;   // 4352-byte blocks per copy
    uint8_t* staging = nullptr;  // one canonical expert, for host sources
    int last_T = -1;
    cudaStream_t last_stream = nullptr;
    // profiling: a ring of event sets, folded into totals when recycled
    static constexpr int kRing = 64;
    bool profiling = false;
    int prof_next = 0;                 // ring slot of the next forward
    int64_t prof_issued = 0;           // forwards recorded since enable
    int64_t prof_folded = 0;           // forwards folded into the totals
    double prof_total[COLI_N_STAGES] = {};
    cudaEvent_t ev[kRing][COLI_N_STAGES + 1] = {};
    int prof_seq[kRing][COLI_N_STAGES] = {};  // stages marked in each ring slot, in the order marked
    int prof_n[kRing] = {};
    // expert cache (coli_moe_layer_create_cached): `cache.slots` routed experts in HBM
    // (slots 0..R-1, the shared experts after them), all E in page-locked host memory
    bool cached = false;
    ExpertCache cache;
    uint8_t* host_pool = nullptr;     // [E][expert_stride] device-layout bytes of every routed expert
    uint8_t* repack_buf = nullptr;    // device: one expert, repacked before it goes to the host pool
    int32_t* slot_dev = nullptr;      // [E + S] weight slot of each expert, read by the kernels
    int32_t* slot_pin = nullptr;      // page-locked staging of that table
    int32_t* ids_pin = nullptr;       // page-locked [max_tokens][K]: the batch's routed ids
    int32_t* ahead_pin = nullptr;     // page-locked [max_tokens][K]: ids predicted by the previous layer
    bool table_dirty = false;         // the host table changed since it was last uploaded
    bool ahead_valid = false;         // ahead_pin holds a prediction for the next forward
    int ahead_T = 0;
    bool lookahead = true;            // accept predictions from the previous layer of a stack
    cudaStream_t copy_stream = nullptr;   // prefetch copies
    cudaEvent_t ev_table = nullptr;       // last upload of the table finished
    cudaEvent_t ev_prefetch = nullptr;    // prefetch copies finished
    cudaEvent_t ev_done = nullptr;        // the last forward's kernels finished reading the slots
    std::vector<char> prefetched;     // [E] resident because of a prefetch, not yet needed
    // expert parallelism (coli_moe_layer_create_ep): this rank's routed experts [ep_lo, ep_hi)
    // in slots 0.., its shared experts (rank 0: all, else none) after them
    bool ep = false;
    int ep_lo = 0, ep_hi = 0;
    int64_t bytes_h2d = 0, n_prefetched = 0, prefetch_used = 0, predicted = 0, predicted_of = 0;
};

// Adds the durations of ring slot `r` to the totals (waits for its last
// event). A stage runs from its mark to the next mark recorded after it (or
// the end mark); stages a path does not run are not marked and add nothing.
static cudaError_t prof_fold(coli_moe_layer* L, int r) {
    cudaError_t e = cudaEventSynchronize(L->ev[r][COLI_N_STAGES]);
    if (e != cudaSuccess) return e;
    const int n = L->prof_n[r];
    for (int k = 0; k < n; ++k) {
        const int i = L->prof_seq[r][k], j = k + 1 < n ? L->prof_seq[r][k + 1] : COLI_N_STAGES;
        float ms = 0.0f;
        e = cudaEventElapsedTime(&ms, L->ev[r][i], L->ev[r][j]);
        if (e != cudaSuccess) return e;
        L->prof_total[i] += ms;
    }
    L->prof_folded += 1;
    return cudaSuccess;
}

// Records the boundary before stage `i` of the current forward
// (i == COLI_N_STAGES: after the last stage). Each stage is marked at most
// once per forward.
static void prof_mark(coli_moe_layer* L, int i, cudaStream_t s) {
    if (!L->profiling) return;
    cudaEventRecord(L->ev[L->prof_next][i], s);
    if (i < COLI_N_STAGES) L->prof_seq[L->prof_next][L->prof_n[L->prof_next]++] = i;
}

static coli_status check_cfg(const coli_moe_config* c) {
    if (!c) return fail(COLI_EINVAL, "config is NULL");
    if (c->hidden <= 0 || c->hidden % 128) return fail(COLI_EINVAL, "hidden must be a positive multiple of 128");
    if (c->inter <= 0 || c->inter % 64) return fail(COLI_EINVAL, "inter must be a positive multiple of 64");
    if (c->group_size != 64) return fail(COLI_EINVAL, "group_size must be 64");
    if (c->n_experts < 1 || c->n_experts > 1024) return fail(COLI_EINVAL, "n_experts must be in [1, 1024]");
    if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > 32) return fail(COLI_EINVAL, "top_k must be in [1, min(n_experts, 32)]");
    if (c->n_shared < 0 || c->n_shared > 64) return fail(COLI_EINVAL, "n_shared must be in [0, 64]");
    if (c->max_tokens < 1 || c->max_tokens > (1 << 20)) return fail(COLI_EINVAL, "max_tokens must be in [1, 2^20]");
    if ((int64_t)c->max_tokens * c->top_k > (1 << 24)) return fail(COLI_EINVAL, "max_tokens * top_k too large");
    return COLI_OK;
}

static void free_layer(coli_moe_layer* L) {
    if (!L) return;
    if (L->weights) cudaFree(L->weights);
    if (L->router_w) cudaFree(L->router_w);
    if (L->router_b) cudaFree(L->router_b);
    if (L->ws) cudaFree(L->ws);
    if (L->staging) cudaFree(L->staging);
    if (L->repack_buf) cudaFree(L->repack_buf);
    if (L->slot_dev) cudaFree(L->slot_dev);
    if (L->host_pool) cudaFreeHost(L->host_pool);
    if (L->slot_pin) cudaFreeHost(L->slot_pin);
    if (L->ids_pin) cudaFreeHost(L->ids_pin);
    if (L->ahead_pin) cudaFreeHost(L->ahead_pin);
    if (L->copy_stream) cudaStreamDestroy(L->copy_stream);
    for (cudaEvent_t e : {L->ev_table, L->ev_prefetch, L->ev_done})
        if (e) cudaEventDestroy(e);
    for (auto& set : L->ev)
        for (auto& e : set)
            if (e) cudaEventDestroy(e);
    delete L;
}

COLI_API coli_status coli_moe_debug_fail_alloc(int nth) {
    if (nth < 0) return fail(COLI_EINVAL, "nth must be >= 0");
    g_fail_alloc.store(nth);
    return COLI_OK;
}

// Weight slot of expert e (routed 0..E-1, shared E..E+S-1): its id, or in a
// cached layer its cache slot (-1: not resident) and R + j for shared expert j.
static int weight_slot(const coli_moe_layer* L, int e) {
    if (L->ep) {  // -1: held by another rank
        if (e < L->d.E) return (e >= L->ep_lo && e < L->ep_hi) ? e - L->ep_lo : -1;
        return e - L->d.E < L->d.S ? (L->ep_hi - L->ep_lo) + (e - L->d.E) : -1;
    }
    if (!L->cached) return e;
    return e < L->d.E ? L->cache.slot(e) : L->cache.slots + (e - L->d.E);
}

// Uploads a cached layer's slot table on stream s if it changed since the
// last upload. Experts that are not resident map to slot 0, an in-bounds
// placeholder: every expert a batch routes to is made resident first. The
// page-locked staging copy is rewritten only after its previous upload ended.
static cudaError_t upload_table(coli_moe_layer* L, cudaStream_t s) {
    if (!L->table_dirty) return cudaSuccess;
    cudaError_t e = cudaEventSynchronize(L->ev_table);
    if (e != cudaSuccess) return e;
    const int E = L->d.E, S = L->d.S;
    for (int i = 0; i < E; ++i) L->slot_pin[i] = std::max(L->cache.slot(i), 0);
    for (int j = 0; j < S; ++j) L->slot_pin[E + j] = L->cache.slots + j;
    e = cudaMemcpyAsync(L->slot_dev, L->slot_pin, (size_t)(E + S) * 4, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return e;
    L->table_dirty = false;
    return cudaEventRecord(L->ev_table, s);
}

COLI_API int64_t coli_moe_expert_bytes(int hidden, int inter) {
    return 3LL * hidden * inter / 2 + 3LL * hidden * inter / 64 * 2;
}

COLI_API coli_status coli_moe_layer_set_experts(coli_moe_layer* L, int first, int count, const uint8_t* q,
                                                const uint16_t* scales) {
    if (!L || !q || !scales) return fail(COLI_EINVAL, "NULL layer or weights");
    const int total = L->cfg.n_experts + L->cfg.n_shared;
    if (first < 0 || count < 0 || first + count > total) return fail(COLI_EINVAL, "expert range out of bounds");
    if (((uintptr_t)scales) & 1u) return fail(COLI_EINVAL, "scales must be 2-byte aligned");
    DeviceGuard guard(L->device);
    if (!guard.ok) return fail(COLI_ECUDA, "cudaSetDevice failed");
    const int H = L->d.H, I = L->d.I;
    const size_t nq = 3ull * H * I / 2, ns = 3ull * H * I / 64;
    const size_t mq = (size_t)I * H / 2, ms = (size_t)I * H / 64;
    // device sources are read in place when 16-byte aligned; anything else goes through the staging buffer
    const bool dev_q = is_device_ptr(q) && ((uintptr_t)q & 15u) == 0, dev_s = is_device_ptr(scales);
    if (L->cached) CUDA_TRY(cudaDeviceSynchronize(), "wait for expert copies");  // nothing reads the pool meanwhile
    for (int i = 0; i < count; ++i) {
        const uint8_t* eq = q + (size_t)i * nq;
        const uint16_t* es = scales + (size_t)i * ns;
        if (!dev_q || !dev_s) {
            if (!L->staging) {
                cudaError_t e = dev_alloc(&L->staging, align256(nq) + ns * 2);
                if (e == cudaErrorMemoryAllocation) return fail(COLI_ENOMEM, "cudaMalloc(staging): out of memory");
                if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(staging)");
            }
            CUDA_TRY(cudaMemcpy(L->staging, eq, nq, cudaMemcpyDefault), "copy expert nibbles");
            CUDA_TRY(cudaMemcpy(L->staging + align256(nq), es, ns * 2, cudaMemcpyDefault), "copy expert scales");
            eq = L->staging;
            es = reinterpret_cast<const uint16_t*>(L->staging + align256(nq));
        }
        // a cached layer's routed expert is repacked once, then kept in the host pool
        const int e = first + i;
        if (L->ep && weight_slot(L, e) < 0) continue;  // another rank's expert
        const bool pooled = L->cached && e < L->d.E;
        uint8_t* dst = pooled ? L->repack_buf : L->weights + (size_t)weight_slot(L, e) * L->d.expert_stride;
        CUDA_TRY(launch_repack(eq, es, eq + mq, es + ms, 2 * I, H, true, dst, 0), "repack gate/up");
        CUDA_TRY(launch_repack(eq + 2 * mq, es + 2 * ms, nullptr, nullptr, H, I, false, dst + L->d.gu_bytes, 0),
                 "repack down");
        CUDA_TRY(launch_l1_bound(eq, es, H, I, L->meta, 0), "weight bounds");
        if (pooled) {
            const size_t stride = (size_t)L->d.expert_stride;
            CUDA_TRY(cudaMemcpy(L->host_pool + (size_t)e * stride, dst, stride, cudaMemcpyDeviceToHost), "expert to host pool");
            const int sl = L->cache.slot(e);
            if (sl >= 0)
                CUDA_TRY(cudaMemcpy(L->weights + (size_t)sl * stride, dst, stride, cudaMemcpyDeviceToDevice),
                         "expert to its slot");
        }
        if (!dev_q || !dev_s) CUDA_TRY(cudaDeviceSynchronize(), "repack");  // staging is reused
    }
    CUDA_TRY(cudaDeviceSynchronize(), "repack");
    unsigned meta[2] = {0, 0};
    CUDA_TRY(cudaMemcpy(meta, L->meta, sizeof meta, cudaMemcpyDeviceToHost), "read weight bounds");
    float max_scale;
    memcpy(&max_scale, &meta[1], 4);
    // fp16 products q * scale (|q| <= 8) stay finite for |scale| <= 4096
    L->tc_scale_ok = max_scale <= 4096.0f;
    return COLI_OK;
}

// resident < 0: every expert in HBM; otherwise an expert cache of `resident` routed slots.
// ep_world > 0: expert parallelism, this layer holding rank ep_rank's share (no cache).
static coli_status create_impl(const coli_moe_config* cfg, const float* router_w, const float* router_bias,
                               const uint8_t* expert_q, const uint16_t* expert_scales, const uint8_t* shared_q,
                               const uint16_t* shared_scales, int resident, int device, coli_moe_layer** out,
                               int ep_rank = 0, int ep_world = 0) {
    if (!out) return fail(COLI_EINVAL, "out is NULL");
    *out = nullptr;
    coli_status st = check_cfg(cfg);
    if (st != COLI_OK) return st;
    if (!router_w) return fail(COLI_EINVAL, "router_w is NULL");
    if ((expert_q == nullptr) != (expert_scales == nullptr)) return fail(COLI_EINVAL, "expert_q/expert_scales: both or neither");
    if ((shared_q == nullptr) != (shared_scales == nullptr)) return fail(COLI_EINVAL, "shared_q/shared_scales: both or neither");
    if (cfg->n_shared == 0 && shared_q) return fail(COLI_EINVAL, "shared weights given with n_shared == 0");
    if (resident >= 0) {
        const int64_t need = std::min<int64_t>((int64_t)cfg->max_tokens * cfg->top_k, cfg->n_experts);
        if (resident < need || resident > cfg->n_experts)
            return fail(COLI_EINVAL, "resident_slots must be in [min(n_experts, max_tokens * top_k), n_experts]");
        if (!expert_q) return fail(COLI_EINVAL, "a cached layer needs expert_q and expert_scales");
    }
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || device < 0 || device >= ndev) {
        cudaGetLastError();
        return fail(COLI_EINVAL, "no such CUDA device");
    }
    DeviceGuard guard(device);
    if (!guard.ok) return fail(COLI_ECUDA, "cudaSetDevice failed");

    coli_moe_layer* L = new (std::nothrow) coli_moe_layer();
    if (!L) return fail(COLI_ENOMEM, "host allocation failed");
    L->cfg = *cfg;
    L->device = device;
    Dims& d = L->d;
    d.H = cfg->hidden; d.I = cfg->inter; d.E = cfg->n_experts; d.K = cfg->top_k; d.S = cfg->n_shared;
    L->ep_hi = d.E;
    if (ep_world > 0) {  // rank r holds [E r / world, E (r + 1) / world) and, on rank 0, the shared experts
        L->ep = true;
        L->ep_lo = (int)((int64_t)d.E * ep_rank / ep_world);
        L->ep_hi = (int)((int64_t)d.E * (ep_rank + 1) / ep_world);
        if (ep_rank != 0) d.S = 0;
    }
    d.max_tokens = cfg->max_tokens;
    d.gu_bytes = matrix_bytes(2 * d.I, d.H);
    d.d_bytes = matrix_bytes(d.H, d.I);
    d.expert_stride = (int64_t)align256((size_t)(d.gu_bytes + d.d_bytes));
    cudaDeviceGetAttribute(&L->n_sm, cudaDevAttrMultiProcessorCount, device);
    int cc_major = 0, optin = 0;
    cudaDeviceGetAttribute(&cc_major, cudaDevAttrComputeCapabilityMajor, device);
    cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
    const int Tm = d.max_tokens;
    L->max_active = (int)std::min<int64_t>((int64_t)Tm * d.K, d.E) + d.S;

    auto bail = [&](cudaError_t e, const char* where) {
        coli_status s = (e == cudaErrorMemoryAllocation) ? fail(COLI_ENOMEM, where) : cuda_fail(e, where);
        cudaGetLastError();
        free_layer(L);
        return s;
    };
    cudaError_t e;
    const size_t n_slots = (size_t)(resident >= 0 ? resident : L->ep_hi - L->ep_lo) + d.S;
    if ((e = dev_alloc(&L->weights, n_slots * d.expert_stride)) != cudaSuccess) return bail(e, "cudaMalloc(weights)");
    if ((e = dev_alloc(&L->router_w, (size_t)d.E * d.H * 4)) != cudaSuccess) return bail(e, "cudaMalloc(router)");
    if ((e = dev_alloc(&L->router_b, (size_t)d.E * 4)) != cudaSuccess) return bail(e, "cudaMalloc(bias)");

    // workspace
    const size_t TE = (size_t)Tm * d.E;
    // batches of kRouterGemmMinTok tokens and more take the certified integer-MMA router when
    // the shapes and the device allow it; the split fp64 GEMM and its partial sums serve the others
    const bool cert = Tm >= kRouterGemmMinTok && router_certified_supported(d.H, d.E) && cc_major == 10 &&
                      (size_t)optin >= router_certified_smem_bytes();
    const size_t rpart_cap = cert ? 0 : std::max<size_t>(TE, std::min<size_t>(64 * TE, (size_t)1 << 23));  // <= 64 MB unless TE is larger
    const size_t TK = (size_t)Tm * d.K, slots = TK + (size_t)d.S * Tm, EA = (size_t)d.E + d.S;
    // the integer-MMA kernel's batches: up to kI8MaxTok tokens and kI8MaxSlots routed slots
    const int Tf = (int)std::min<int64_t>(std::min<int64_t>(Tm, kI8MaxTok), kI8MaxSlots / d.K);
    L->i8_max_tok = Tf;
    const size_t slots_f = (size_t)Tf * d.K + (size_t)d.S * Tf;
    L->ctl_n = std::max(kCtlError + 1, Tf > 0 ? i8_ctl_ints_for(d, Tf) : 0);
    size_t sz[] = {Tm * (size_t)d.E * 8, TK * 4, TK * 4, (size_t)d.E * 4, (size_t)(d.E + 1) * 4, (size_t)d.E * 4, 4,
                   TK * 4, slots * 4, EA * 4, EA * 4, EA * 4, 4, slots * d.I * 4, slots * d.H * 4, (size_t)Tm * d.H * 4,
                   (size_t)L->ctl_n * 4, 0, 2 * slots * d.H * 2, (size_t)Tm * 16,
                   slots * 16, (size_t)prefill_tc_max_tiles(d, Tm) * 16, 4, 16, rpart_cap * 8, (EA + 1) * 4,
                   (size_t)Tf * (d.H / 64) * 128, (size_t)Tf * (d.H / 64) * 16, slots_f * (d.I / 64) * 128,
                   slots_f * (d.I / 64) * 16,
                   // certified router: batch digit planes, token scales, fallback list, token norms,
                   // router digit planes, expert scales, expert bound factors
                   cert ? (size_t)4 * Tm * d.H : 0, cert ? (size_t)Tm * 4 : 0, cert ? (size_t)(Tm + 1) * 4 : 0,
                   cert ? (size_t)Tm * 24 : 0, cert ? (size_t)4 * d.E * d.H : 0, cert ? (size_t)d.E * 4 : 0,
                   cert ? (size_t)d.E * 24 : 0};
    constexpr int kRegions = sizeof(sz) / sizeof(sz[0]);
    size_t total = 0;
    for (size_t s : sz) total += align256(s);
    if ((e = dev_alloc(&L->ws, total)) != cudaSuccess) return bail(e, "cudaMalloc(workspace)");
    L->ws_bytes = total;
    uint8_t* cur = L->ws;
    void* ptrs[kRegions];
    for (int i = 0; i < kRegions; ++i) { ptrs[i] = cur; cur += align256(sz[i]); }
    L->ctl = (int*)ptrs[16];
    L->xs = (__half*)ptrs[18];
    L->tscale = (float4*)ptrs[19];
    L->slot = (float4*)ptrs[20];
    L->tiles = (int4*)ptrs[21];
    L->n_tiles = (int*)ptrs[22];
    L->meta = (unsigned*)ptrs[23];
    L->rpart = (double*)ptrs[24];
    L->plan.act_chunk = (int32_t*)ptrs[25];
    L->xq = (uint8_t*)ptrs[26];
    L->xm = (uint8_t*)ptrs[27];
    L->hq = (uint8_t*)ptrs[28];
    L->hm = (uint8_t*)ptrs[29];
    L->rc.maps = L->rc_maps;
    L->rc.xd8 = (uint8_t*)ptrs[30];
    L->rc.xscale = (int*)ptrs[31];
    L->rc.fail = (int*)ptrs[32];
    L->rc.xb = (double*)ptrs[33];
    L->rc.wd8 = (uint8_t*)ptrs[34];
    L->rc.wscale = (int*)ptrs[35];
    L->rc.wb = (double*)ptrs[36];
    L->rc.Tm = Tm;
    L->rc.H = d.H;
    L->rc.E = d.E;
    L->rc.n_sm = L->n_sm;
    L->cert_ok = cert;
    L->rpart_cap = rpart_cap;
    {
        L->smem_optin = (size_t)optin;
        L->fused = (Tf > 0 && decode_i8_supported(d, 1, L->smem_optin)) ? 1 : 0;
        L->tc_shape_ok = cc_major == 10 && d.H % 256 == 0 && d.I % 128 == 0 && L->smem_optin >= prefill_tc_smem_bytes();
    }
    if (L->tc_shape_ok) {
        // xs [slots][H] and h16 [slots][I] (in the h region) as token operands
        if (make_token_map(L->xs_maps, ptrs[18], 2 * (int)slots, d.H, kTcMaxTok) != cudaSuccess ||
            make_token_map(L->xs_maps + kTensorMapBytes, ptrs[18], 2 * (int)slots, d.H, 32) != cudaSuccess ||
            make_token_map(L->h16_maps, ptrs[13], (int)slots, d.I, kTcMaxTok) != cudaSuccess ||
            make_token_map(L->h16_maps + kTensorMapBytes, ptrs[13], (int)slots, d.I, 32) != cudaSuccess) {
            cudaGetLastError();
            L->tc_shape_ok = false;
        }
    }
    L->logits = (double*)ptrs[0];
    Plan& p = L->plan;
    p.ids = (int32_t*)ptrs[1]; p.w = (float*)ptrs[2]; p.cnt = (int32_t*)ptrs[3]; p.off = (int32_t*)ptrs[4];
    p.unique = (int32_t*)ptrs[5]; p.n_unique = (int32_t*)ptrs[6]; p.pos = (int32_t*)ptrs[7]; p.tok = (int32_t*)ptrs[8];
    p.act_expert = (int32_t*)ptrs[9]; p.act_off = (int32_t*)ptrs[10]; p.act_cnt = (int32_t*)ptrs[11];
    p.n_active = (int32_t*)ptrs[12];
    L->h = (float*)ptrs[13]; L->o = (float*)ptrs[14]; L->xn = (float*)ptrs[15];
    if ((e = cudaMemset(L->ws, 0, total)) != cudaSuccess) return bail(e, "cudaMemset(workspace)");
    if ((e = cudaMemset(L->weights, 0, n_slots * d.expert_stride)) != cudaSuccess) return bail(e, "cudaMemset(weights)");
    if (resident >= 0) {
        // the backing store of every routed expert, page-locked, and the slot table
        L->cached = true;
        L->cache.init(d.E, resident);
        L->prefetched.assign(d.E, 0);
        const size_t TKm = (size_t)Tm * d.K;
        if ((e = dev_alloc(&L->repack_buf, (size_t)d.expert_stride)) != cudaSuccess) return bail(e, "cudaMalloc(repack)");
        if ((e = dev_alloc(&L->slot_dev, EA * 4)) != cudaSuccess) return bail(e, "cudaMalloc(slot table)");
        if ((e = host_alloc(&L->host_pool, (size_t)d.E * d.expert_stride)) != cudaSuccess) return bail(e, "cudaHostAlloc(expert pool)");
        if ((e = host_alloc(&L->slot_pin, EA * 4)) != cudaSuccess) return bail(e, "cudaHostAlloc(slot table)");
        if ((e = host_alloc(&L->ids_pin, TKm * 4)) != cudaSuccess) return bail(e, "cudaHostAlloc(ids)");
        if ((e = host_alloc(&L->ahead_pin, TKm * 4)) != cudaSuccess) return bail(e, "cudaHostAlloc(lookahead ids)");
        if ((e = cudaStreamCreateWithFlags(&L->copy_stream, cudaStreamNonBlocking)) != cudaSuccess) return bail(e, "copy stream");
        for (cudaEvent_t* ev : {&L->ev_table, &L->ev_prefetch, &L->ev_done})
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return bail(e, "cudaEventCreate");
        L->table_dirty = true;
        if ((e = upload_table(L, nullptr)) != cudaSuccess) return bail(e, "upload slot table");
        d.slot_of = L->slot_dev;
    }
    if (L->ep) {  // slot table of this rank's experts (others: slot 0, never read)
        std::vector<int32_t> table(EA, 0);
        for (int x = 0; x < (int)EA; ++x) table[x] = std::max(weight_slot(L, x), 0);
        if ((e = dev_alloc(&L->slot_dev, EA * 4)) != cudaSuccess) return bail(e, "cudaMalloc(slot table)");
        if ((e = cudaMemcpy(L->slot_dev, table.data(), EA * 4, cudaMemcpyHostToDevice)) != cudaSuccess)
            return bail(e, "upload slot table");
        d.slot_of = L->slot_dev;
    }

    if ((e = cudaMemcpy(L->router_w, router_w, (size_t)d.E * d.H * 4, cudaMemcpyDefault)) != cudaSuccess) return bail(e, "copy router");
    if (router_bias) {
        if ((e = cudaMemcpy(L->router_b, router_bias, (size_t)d.E * 4, cudaMemcpyDefault)) != cudaSuccess) return bail(e, "copy bias");
    } else if ((e = cudaMemset(L->router_b, 0, (size_t)d.E * 4)) != cudaSuccess) {
        return bail(e, "clear bias");
    }
    if (L->cert_ok && (e = router_certified_prepare(L->rc, L->router_w, nullptr)) != cudaSuccess)
        return bail(e, "router digit planes");
    if (expert_q) {
        st = coli_moe_layer_set_experts(L, 0, d.E, expert_q, expert_scales);
        if (st != COLI_OK) { free_layer(L); return st; }
    }
    if (shared_q && d.S > 0) {
        st = coli_moe_layer_set_experts(L, d.E, d.S, shared_q, shared_scales);
        if (st != COLI_OK) { free_layer(L); return st; }
    }
    if ((e = cudaDeviceSynchronize()) != cudaSuccess) return bail(e, "create");
    *out = L;
    return COLI_OK;
}

COLI_API coli_status coli_moe_layer_create(const coli_moe_config* cfg, const float* router_w, const float* router_bias,
                                           const uint8_t* expert_q, const uint16_t* expert_scales,
                                           const uint8_t* shared_q, const uint16_t* shared_scales, int device,
                                           coli_moe_layer** out) {
    return create_impl(cfg, router_w, router_bias, expert_q, expert_scales, shared_q, shared_scales, -1, device, out);
}

COLI_API coli_status coli_moe_ep_range(int n_experts, int rank, int world, int* first, int* end) {
    if (n_experts < 1 || world < 1 || rank < 0 || rank >= world || !first || !end)
        return fail(COLI_EINVAL, "need n_experts >= 1, 0 <= rank < world, non-NULL outputs");
    *first = (int)((int64_t)n_experts * rank / world);
    *end = (int)((int64_t)n_experts * (rank + 1) / world);
    return COLI_OK;
}

COLI_API coli_status coli_moe_layer_create_ep(const coli_moe_config* cfg, const float* router_w,
                                              const float* router_bias, const uint8_t* expert_q,
                                              const uint16_t* expert_scales, const uint8_t* shared_q,
                                              const uint16_t* shared_scales, int rank, int world, int device,
                                              coli_moe_layer** out) {
    if (out) *out = nullptr;
    if (!cfg || world < 1 || rank < 0 || rank >= world || world > cfg->n_experts)
        return fail(COLI_EINVAL, "need 1 <= world <= n_experts and 0 <= rank < world");
    return create_impl(cfg, router_w, router_bias, expert_q, expert_scales, shared_q, shared_scales, -1, device, out,
                       rank, world);
}

COLI_API coli_status coli_moe_layer_create_cached(const coli_moe_config* cfg, const float* router_w,
                                                  const float* router_bias, const uint8_t* expert_q,
                                                  const uint16_t* expert_scales, const uint8_t* shared_q,
                                                  const uint16_t* shared_scales, int resident_slots, int device,
                                                  coli_moe_layer** out) {
    if (resident_slots < 0) {
        if (out) *out = nullptr;
        return fail(COLI_EINVAL, "resident_slots must be >= 0");
    }
    return create_impl(cfg, router_w, router_bias, expert_q, expert_scales, shared_q, shared_scales, resident_slots,
                       device, out);
}

COLI_API void coli_moe_layer_destroy(coli_moe_layer* L) {
    if (!L) return;
    DeviceGuard guard(L->device);
    cudaDeviceSynchronize();
    free_layer(L);
}

COLI_API coli_status coli_moe_layer_config(const coli_moe_layer* L, coli_moe_config* cfg) {
    if (!L || !cfg) return fail(COLI_EINVAL, "NULL argument");
    *cfg = L->cfg;
    return COLI_OK;
}

static coli_status check_call(const coli_moe_layer* L, const void* x, coli_dtype dt, int T) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (dt != COLI_F32 && dt != COLI_BF16) return fail(COLI_EINVAL, "dtype must be COLI_F32 or COLI_BF16");
    if (T < 0 || T > L->cfg.max_tokens) return fail(COLI_EINVAL, "n_tokens out of [0, max_tokens]");
    if (T > 0 && !x) return fail(COLI_EINVAL, "x is NULL");
    if (((uintptr_t)x) & 15u) return fail(COLI_EINVAL, "x must be 16-byte aligned");
    return COLI_OK;
}

// Router and top-K of a batch into ids/weights: batches of kRouterGemmMinTok
// tokens and more take the certified integer-MMA router (fp64 only where the
// bounds do not settle the selection), smaller ones the fp64 GEMV and top-K.
// Returns the number of kernels enqueued, or -1 on a launch error.
static int route_batch(coli_moe_layer* L, const void* x, coli_dtype dt, int T, int32_t* ids, float* w, int e_lo,
                       int e_hi, cudaStream_t s) {
    const Dims& d = L->d;
    if (L->cert_ok && T >= kRouterGemmMinTok) {
        if (launch_router_certified(L->rc, L->router_w, L->router_b, x, dt, T, d.K, L->topp, e_lo, e_hi, L->logits, ids,
                                    w, L->ctl + kCtlError, L->wait_ns, L->wait_test, s) != cudaSuccess)
            return -1;
        return 5;
    }
    if (launch_router_logits(L->router_w, L->router_b, x, dt, T, d.H, d.E, L->logits, s, L->rpart, L->rpart_cap) !=
            cudaSuccess ||
        launch_topk(L->logits, T, d.E, d.K, ids, w, s, L->topp, e_lo, e_hi) != cudaSuccess)
        return -1;
    return router_kernel_count(T, d.H, d.E, L->rpart, L->rpart_cap) + 1;
}

COLI_API coli_status coli_moe_route(coli_moe_layer* L, const void* x, coli_dtype dt, int T, int32_t* ids,
                                    float* weights, coli_stream stream) {
    coli_status st = check_call(L, x, dt, T);
    if (st != COLI_OK) return st;
    if (T > 0 && (!ids || !weights)) return fail(COLI_EINVAL, "ids/weights is NULL");
    if (T == 0) return COLI_OK;
    DeviceGuard guard(L->device);
    cudaStream_t s = (cudaStream_t)stream;
    const int n = route_batch(L, x, dt, T, ids, weights, 0, L->d.E, s);
    if (n < 0) return cuda_fail(cudaGetLastError(), "router");
    L->launches += n;
    return COLI_OK;
}

// Starts the profile record of a forward (recycles the oldest ring slot).
static coli_status prof_begin(coli_moe_layer* L) {
    if (!L->profiling) return COLI_OK;
    if (L->prof_issued - L->prof_folded >= coli_moe_layer::kRing) CUDA_TRY(prof_fold(L, L->prof_next), "profile");
    L->prof_n[L->prof_next] = 0;
    return COLI_OK;
}

// x: layer input; residual: added to the output (stack) or NULL; y: output.
// routed: the plan's ids and weights already hold this batch's routing (and
// the caller began the profile record), so the router and top-k do not run.
static coli_status forward_impl(coli_moe_layer* L, const void* x, void* y, coli_dtype dt, int T, const float* residual,
                                cudaStream_t s, bool routed = false) {
    const Dims& d = L->d;
    const Plan& p = L->plan;
    if (!routed) {
        coli_status st = prof_begin(L);
        if (st != COLI_OK) return st;
    }
    if (L->fused == 1 && T <= L->i8_max_tok && decode_i8_supported(d, T, L->smem_optin)) {
        prof_mark(L, COLI_STAGE_FUSED, s);
        I8Launch l{};
        l.weights = L->weights; l.d = d; l.wr = L->router_w; l.bias = L->router_b; l.x = x; l.dt = dt; l.T = T;
        l.y = y; l.residual = residual; l.p = p; l.logits = L->logits; l.xq = L->xq; l.xm = L->xm; l.hq = L->hq;
        l.hm = L->hm; l.o = L->o; l.ctl = L->ctl; l.n_sm = L->n_sm; l.smem_limit = L->smem_optin; l.trace = L->trace;
        l.trace_cap = L->trace_cap; l.max_stages = L->ring_stages; l.max_sb = L->ring_blocks;
        l.wait_ns = L->wait_ns; l.wait_test = L->wait_test;
        l.topp = L->topp;
        l.ep_lo = L->ep_lo;
        l.ep_hi = L->ep_hi;
        if (routed) { l.given_ids = p.ids; l.given_w = p.w; }
        CUDA_TRY(launch_decode_i8(l, s), "persistent decode kernel (integer MMA)");
        L->launches += 1;
    } else if ((L->tc_mode == 2 || (L->tc_mode == 1 && dt == COLI_BF16)) && L->tc_shape_ok && L->tc_scale_ok) {
        // tensor cores; fp32 tokens as fp16 hi + lo operand rows (tiles of kTcMaxTok / 2 tokens)
        const bool pairs = dt == COLI_F32;
        if (!routed) {
            prof_mark(L, COLI_STAGE_ROUTER, s);
            const int n = route_batch(L, x, dt, T, p.ids, p.w, L->ep_lo, L->ep_hi, s);
            if (n < 0) return cuda_fail(cudaGetLastError(), "router");
            L->launches += n;
        }
        prof_mark(L, COLI_STAGE_PLAN, s);
        CUDA_TRY(launch_plan(p.ids, T, d.K, d.E, d.S, p, s), "plan");
        // the plan stage also covers the operand rows, the tile list and the output clear,
        // so the gate/up and down stages time the grouped GEMMs alone
        __half* h16 = reinterpret_cast<__half*>(L->h);
        CUDA_TRY(launch_prefill_prep(x, dt, T, d.H, d.K, d.S, p.pos, reinterpret_cast<const float*>(L->meta), L->xs,
                                     L->tscale, s),
                 "prep");
        CUDA_TRY(launch_prefill_plan(p, T, d.K, d.S, pairs ? kTcMaxTok / 2 : kTcMaxTok, L->tscale, L->slot, L->tiles,
                                     L->n_tiles, s),
                 "tile plan");
        CUDA_TRY(cudaMemsetAsync(L->o, 0, (size_t)T * d.H * 4, s), "clear output");
        prof_mark(L, COLI_STAGE_GATEUP, s);
        // with a trace buffer: block timeline of the gate/up launch, then of the down launch
        const int tcap = L->trace ? (L->trace_cap - 256) / 16 : 0;
        CUDA_TRY(launch_prefill_gemm(0, pairs, L->weights, d, L->xs_maps, p, L->slot, L->tiles, L->n_tiles, h16, nullptr,
                                     L->ctl + kCtlError, L->n_sm, tcap > 0 ? L->trace : nullptr, tcap, L->wait_ns,
                                     L->wait_test, s),
                 "gate/up (tensor cores)");
        prof_mark(L, COLI_STAGE_DOWN, s);
        CUDA_TRY(launch_prefill_gemm(1, false, L->weights, d, L->h16_maps, p, L->slot, L->tiles, L->n_tiles, nullptr,
                                     L->o, L->ctl + kCtlError, L->n_sm,
                                     tcap > 0 ? L->trace + (size_t)tcap * 8 + 128 : nullptr, tcap, L->wait_ns, L->wait_test, s),
                 "down (tensor cores)");
        prof_mark(L, COLI_STAGE_COMBINE, s);
        CUDA_TRY(launch_prefill_out(L->o, residual, T, d.H, y, dt, s), "output");
        // plan, prep, tile plan, two grouped GEMMs, output (the clear is a driver memset; the router counted above)
        L->launches += 6;
    } else {
        if (!routed) {
            prof_mark(L, COLI_STAGE_ROUTER, s);
            const int n = route_batch(L, x, dt, T, p.ids, p.w, L->ep_lo, L->ep_hi, s);
            if (n < 0) return cuda_fail(cudaGetLastError(), "router");
            L->launches += n;
        }
        prof_mark(L, COLI_STAGE_PLAN, s);
        CUDA_TRY(launch_plan(p.ids, T, d.K, d.E, d.S, p, s), "plan");
        prof_mark(L, COLI_STAGE_GATEUP, s);
        CUDA_TRY(launch_gateup_core(L->weights, d, x, dt, T, p, L->h, L->max_active, L->n_sm, s), "gate/up");
        prof_mark(L, COLI_STAGE_DOWN, s);
        CUDA_TRY(launch_down_core(L->weights, d, L->h, T, p, L->o, L->max_active, L->n_sm, s), "down");
        prof_mark(L, COLI_STAGE_COMBINE, s);
        CUDA_TRY(launch_combine(L->o, p, T, d.H, d.K, d.S, residual, y, dt, s), "combine");
        L->launches += 4;
    }
    prof_mark(L, COLI_N_STAGES, s);
    if (L->profiling) {
        L->prof_issued += 1;
        L->prof_next = (L->prof_next + 1) % coli_moe_layer::kRing;
    }
    L->last_T = T;
    L->last_stream = s;
    return COLI_OK;
}

// ---------------------------------------------------------------- expert cache

// Issues one host-to-HBM copy per (expert, slot) pair on stream s: an
// expert's gate/up and down matrices are adjacent, so each is one copy.
static cudaError_t copy_experts(coli_moe_layer* L, const std::vector<std::pair<int, int>>& copies, cudaStream_t s) {
    const size_t stride = (size_t)L->d.expert_stride, bytes = (size_t)(L->d.gu_bytes + L->d.d_bytes);
    for (const auto& c : copies) {
        cudaError_t e = cudaMemcpyAsync(L->weights + (size_t)c.second * stride, L->host_pool + (size_t)c.first * stride,
                                        bytes, cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return e;
        L->bytes_h2d += (int64_t)bytes;
    }
    if (!copies.empty()) L->table_dirty = true;
    return cudaSuccess;
}

// Distinct ids among ids[0..n), in first-appearance order; false if one is
// outside [0, E).
static bool distinct_ids(const int32_t* ids, int n, int E, std::vector<int32_t>* out) {
    std::vector<char> seen(E, 0);
    out->clear();
    for (int i = 0; i < n; ++i) {
        const int e = ids[i];
        if (e < 0 || e >= E) return false;
        if (!seen[e]) {
            seen[e] = 1;
            out->push_back(e);
        }
    }
    return true;
}

// Best-effort prefetch of the distinct experts among ids[0..n) on the copy
// stream, after the layer's last forward has finished reading its slots.
static coli_status cache_prefetch(coli_moe_layer* L, const int32_t* ids, int n) {
    std::vector<int32_t> ex;
    if (!distinct_ids(ids, n, L->d.E, &ex)) return fail(COLI_EINVAL, "expert id out of range");
    std::vector<std::pair<int, int>> copies;
    L->cache.prefetch(ex.data(), (int)ex.size(), &copies);
    for (int e = 0; e < L->d.E; ++e)
        if (L->prefetched[e] && L->cache.slot(e) < 0) L->prefetched[e] = 0;  // evicted before use
    if (copies.empty()) return COLI_OK;
    CUDA_TRY(cudaStreamWaitEvent(L->copy_stream, L->ev_done, 0), "prefetch: wait for the last forward");
    CUDA_TRY(copy_experts(L, copies, L->copy_stream), "prefetch copy");
    CUDA_TRY(cudaEventRecord(L->ev_prefetch, L->copy_stream), "record prefetch");
    for (const auto& c : copies) L->prefetched[c.first] = 1;
    L->n_prefetched += (int64_t)copies.size();
    return COLI_OK;
}

// Makes every routed expert of the batch whose ids are in ids_pin resident:
// misses are copied on stream s after any pending prefetch, then the table.
static coli_status cache_admit(coli_moe_layer* L, int T, cudaStream_t s) {
    const int E = L->d.E, TK = T * L->d.K;
    std::vector<int32_t> ex;
    if (!distinct_ids(L->ids_pin, TK, E, &ex)) return fail(COLI_ECUDA, "routed expert id out of range");
    if (L->ahead_valid) {  // how many of the needed experts the previous layer predicted
        std::vector<char> pred(E, 0);
        for (int i = 0; i < L->ahead_T * L->d.K; ++i) {
            const int e = L->ahead_pin[i];
            if (e >= 0 && e < E) pred[e] = 1;
        }
        for (int e : ex) L->predicted += pred[e];
        L->predicted_of += (int64_t)ex.size();
        L->ahead_valid = false;
    }
    for (int e : ex)
        if (L->prefetched[e] && L->cache.slot(e) >= 0) {
            L->prefetch_used += 1;
            L->prefetched[e] = 0;
        }
    std::vector<std::pair<int, int>> copies;
    if (!L->cache.admit(ex.data(), (int)ex.size(), &copies))
        return fail(COLI_EUNSUPPORTED, "too many pinned experts for this batch");
    for (int e = 0; e < E; ++e)
        if (L->prefetched[e] && L->cache.slot(e) < 0) L->prefetched[e] = 0;
    CUDA_TRY(cudaStreamWaitEvent(s, L->ev_prefetch, 0), "wait for prefetch copies");
    CUDA_TRY(copy_experts(L, copies, s), "copy missing experts");
    CUDA_TRY(upload_table(L, s), "upload slot table");
    return COLI_OK;
}

// Forward of a cached layer: route, read the ids back (waits for them), make
// the batch's experts resident, then the resident layer's kernels with the
// given routing. `next`: the following layer of a stack or NULL; when it is a
// cached layer accepting predictions, its router also runs on this layer's
// input, and the experts it picks are prefetched into it while this layer's
// kernels run.
static coli_status cached_forward(coli_moe_layer* L, const void* x, void* y, coli_dtype dt, int T,
                                  const float* residual, cudaStream_t s, coli_moe_layer* next) {
    const Dims& d = L->d;
    const Plan& p = L->plan;
    coli_status st = prof_begin(L);
    if (st != COLI_OK) return st;
    prof_mark(L, COLI_STAGE_ROUTER, s);
    const int nr = route_batch(L, x, dt, T, p.ids, p.w, L->ep_lo, L->ep_hi, s);
    if (nr < 0) return cuda_fail(cudaGetLastError(), "router");
    L->launches += nr;
    prof_mark(L, COLI_STAGE_CACHE, s);
    const bool ahead = next && next != L && next->cached && next->lookahead && T <= next->cfg.max_tokens &&
                       next->d.H == d.H && next->device == L->device;
    if (ahead) {
        const Dims& dn = next->d;
        const int nn = route_batch(next, x, dt, T, next->plan.ids, next->plan.w, 0, dn.E, s);
        if (nn < 0) return cuda_fail(cudaGetLastError(), "lookahead router");
        next->launches += nn;
        CUDA_TRY(cudaMemcpyAsync(next->ahead_pin, next->plan.ids, (size_t)T * dn.K * 4, cudaMemcpyDeviceToHost, s),
                 "read predicted ids");
    }
    CUDA_TRY(cudaMemcpyAsync(L->ids_pin, p.ids, (size_t)T * d.K * 4, cudaMemcpyDeviceToHost, s), "read routed ids");
    CUDA_TRY(cudaStreamSynchronize(s), "wait for routed ids");
    st = cache_admit(L, T, s);
    if (st != COLI_OK) return st;
    st = forward_impl(L, x, y, dt, T, residual, s, true);
    if (st != COLI_OK) return st;
    CUDA_TRY(cudaEventRecord(L->ev_done, s), "record forward");
    if (ahead) {
        next->ahead_valid = true;
        next->ahead_T = T;
        st = cache_prefetch(next, next->ahead_pin, T * next->d.K);
        if (st != COLI_OK) return st;
    }
    return COLI_OK;
}

COLI_API coli_status coli_moe_forward(coli_moe_layer* L, const void* x, void* y, coli_dtype dt, int T,
                                      coli_stream stream) {
    coli_status st = check_call(L, x, dt, T);
    if (st != COLI_OK) return st;
    if (T > 0 && !y) return fail(COLI_EINVAL, "y is NULL");
    if (((uintptr_t)y) & 15u) return fail(COLI_EINVAL, "y must be 16-byte aligned");
    if (T > 0) {
        const size_t bytes = (size_t)T * L->d.H * (dt == COLI_F32 ? 4 : 2);
        const uint8_t *xb = (const uint8_t*)x, *yb = (const uint8_t*)y;
        if (xb < yb + bytes && yb < xb + bytes) return fail(COLI_EINVAL, "x and y overlap");
    }
    if (T == 0) return COLI_OK;
    DeviceGuard guard(L->device);
    if (L->cached) return cached_forward(L, x, y, dt, T, nullptr, (cudaStream_t)stream, nullptr);
    return forward_impl(L, x, y, dt, T, nullptr, (cudaStream_t)stream);
}

COLI_API coli_status coli_moe_stack_forward(coli_moe_layer* const* layers, int n_layers, float* x, int T, float eps,
                                            coli_stream stream) {
    if (!layers || n_layers < 0) return fail(COLI_EINVAL, "bad layer list");
    if (n_layers == 0 || T == 0) return COLI_OK;
    if (!(eps >= 0.0f)) return fail(COLI_EINVAL, "eps must be >= 0");
    const coli_moe_layer* L0 = layers[0];
    for (int l = 0; l < n_layers; ++l) {
        coli_status st = check_call(layers[l], x, COLI_F32, T);
        if (st != COLI_OK) return st;
        if (layers[l]->d.H != L0->d.H || layers[l]->device != L0->device)
            return fail(COLI_EINVAL, "layers must share hidden size and device");
    }
    DeviceGuard guard(L0->device);
    cudaStream_t s = (cudaStream_t)stream;
    for (int l = 0; l < n_layers; ++l) {
        coli_moe_layer* L = layers[l];
        CUDA_TRY(launch_rmsnorm(x, T, L->d.H, eps, L->xn, s), "rmsnorm");
        L->launches += 1;
        coli_status st = L->cached ? cached_forward(L, L->xn, x, COLI_F32, T, x, s, l + 1 < n_layers ? layers[l + 1] : nullptr)
                                   : forward_impl(L, L->xn, x, COLI_F32, T, x, s);
        if (st != COLI_OK) return st;
    }
    return COLI_OK;
}

// Waits for the layer's last forward and reports a device-side timeout of one
// of its kernels (then clears the control block so the layer stays usable).
static coli_status sync_and_check(coli_moe_layer* L) {
    CUDA_TRY(cudaStreamSynchronize(L->last_stream), "sync");
    int err = 0;
    CUDA_TRY(cudaMemcpy(&err, L->ctl + kCtlError, 4, cudaMemcpyDeviceToHost), "read status");
    if (err != 0) {
        CUDA_TRY(cudaMemset(L->ctl, 0, (size_t)L->ctl_n * 4), "reset control block");
        char msg[96];
        if (err == kCtlErrBufferOverflow)
            snprintf(msg, sizeof msg, "a decode work item exceeded its operand buffer (site %d)", err);
        else
            snprintf(msg, sizeof msg, "a bounded wait in a kernel of this layer timed out (site %d)", err);
        g_last_error = msg;
        return COLI_ECUDA;
    }
    return COLI_OK;
}

COLI_API coli_status coli_moe_sync(coli_moe_layer* L) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (L->last_T < 0) return COLI_OK;
    DeviceGuard guard(L->device);
    return sync_and_check(L);
}

COLI_API coli_status coli_moe_set_fused(coli_moe_layer* L, int enable) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (enable < 0 || enable > 1) return fail(COLI_EINVAL, "enable must be 0 or 1");
    if (enable && !(L->i8_max_tok > 0 && decode_i8_supported(L->d, 1, L->smem_optin)))
        return fail(COLI_EUNSUPPORTED, "shapes too large for the persistent kernel's shared memory");
    L->fused = enable;
    return COLI_OK;
}

COLI_API coli_status coli_moe_set_expert_top_p(coli_moe_layer* L, double p) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!(p > 0.0 && p <= 1.0)) return fail(COLI_EINVAL, "p must be in (0, 1]");
    L->topp = p;
    return COLI_OK;
}

COLI_API coli_status coli_moe_debug_wait_test(coli_moe_layer* L, int enable, int64_t wait_ns) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (wait_ns < 0) return fail(COLI_EINVAL, "wait_ns must be >= 0");
    L->wait_test = enable != 0;
    L->wait_ns = wait_ns;
    return COLI_OK;
}

COLI_API coli_status coli_moe_set_tensor_cores(coli_moe_layer* L, int mode) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (mode < 0 || mode > 2) return fail(COLI_EINVAL, "mode must be 0, 1 or 2");
    if (mode && !L->tc_shape_ok)
        return fail(COLI_EUNSUPPORTED, "tensor-core path needs sm_100, hidden % 256 == 0 and inter % 128 == 0");
    if (mode && !L->tc_scale_ok) return fail(COLI_EUNSUPPORTED, "a weight scale exceeds 4096 in magnitude");
    L->tc_mode = mode;
    return COLI_OK;
}

COLI_API coli_status coli_moe_set_ring(coli_moe_layer* L, int stages, int blocks_per_stage) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (stages < 2 || stages > 24 || blocks_per_stage < 2 || blocks_per_stage > 16 || (blocks_per_stage & 1))
        return fail(COLI_EINVAL, "stages in [2, 24], blocks_per_stage even in [2, 16]");
    L->ring_stages = stages;
    L->ring_blocks = blocks_per_stage;
    return COLI_OK;
}

COLI_API coli_status coli_moe_set_trace(coli_moe_layer* L, void* buffer, int capacity) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (buffer && (capacity < 1 || ((uintptr_t)buffer & 7u))) return fail(COLI_EINVAL, "bad trace buffer");
    L->trace = (long long*)buffer;
    L->trace_cap = buffer ? capacity : 0;
    return COLI_OK;
}

COLI_API coli_status coli_moe_get_stats(coli_moe_layer* L, int* n_unique, int64_t* bytes_streamed,
                                        int32_t* per_expert_counts) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (L->last_T < 0) return fail(COLI_EINVAL, "no forward has run on this layer");
    DeviceGuard guard(L->device);
    {
        coli_status st = sync_and_check(L);
        if (st != COLI_OK) return st;
    }
    int nu = 0;
    CUDA_TRY(cudaMemcpy(&nu, L->plan.n_unique, 4, cudaMemcpyDeviceToHost), "read n_unique");
    if (n_unique) *n_unique = nu;
    if (bytes_streamed)
        *bytes_streamed = (int64_t)(nu + L->d.S) * coli_moe_expert_bytes(L->d.H, L->d.I) + (int64_t)L->d.E * L->d.H * 4;
    if (per_expert_counts)
        CUDA_TRY(cudaMemcpy(per_expert_counts, L->plan.cnt, (size_t)L->d.E * 4, cudaMemcpyDeviceToHost), "read counts");
    return COLI_OK;
}

COLI_API coli_status coli_moe_get_launch_count(const coli_moe_layer* L, int64_t* n) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!n) return fail(COLI_EINVAL, "n is NULL");
    *n = L->launches;
    return COLI_OK;
}

COLI_API coli_status coli_moe_router_fallbacks(coli_moe_layer* L, int32_t* certified, int32_t* n) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (certified) *certified = L->cert_ok ? 1 : 0;
    if (!n) return COLI_OK;
    *n = 0;
    if (!L->cert_ok) return COLI_OK;
    DeviceGuard guard(L->device);
    CUDA_TRY(cudaMemcpy(n, L->rc.fail, 4, cudaMemcpyDeviceToHost), "read fallback count");
    return COLI_OK;
}

COLI_API coli_status coli_moe_get_plan(coli_moe_layer* L, int32_t* ids, float* weights, int32_t* counts, int32_t* offsets,
                                       int32_t* unique, int32_t* n_unique, int32_t* pos, int32_t* tok) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (L->last_T < 0) return fail(COLI_EINVAL, "no forward has run on this layer");
    DeviceGuard guard(L->device);
    {
        coli_status st = sync_and_check(L);
        if (st != COLI_OK) return st;
    }
    const size_t TK = (size_t)L->last_T * L->d.K;
    const Plan& p = L->plan;
    int nu = 0;
    CUDA_TRY(cudaMemcpy(&nu, p.n_unique, 4, cudaMemcpyDeviceToHost), "read n_unique");
    if (n_unique) *n_unique = nu;
    if (ids && TK) CUDA_TRY(cudaMemcpy(ids, p.ids, TK * 4, cudaMemcpyDeviceToHost), "read ids");
    if (weights && TK) CUDA_TRY(cudaMemcpy(weights, p.w, TK * 4, cudaMemcpyDeviceToHost), "read weights");
    if (counts) CUDA_TRY(cudaMemcpy(counts, p.cnt, (size_t)L->d.E * 4, cudaMemcpyDeviceToHost), "read counts");
    if (offsets) CUDA_TRY(cudaMemcpy(offsets, p.off, (size_t)(L->d.E + 1) * 4, cudaMemcpyDeviceToHost), "read offsets");
    if (unique && nu) CUDA_TRY(cudaMemcpy(unique, p.unique, (size_t)nu * 4, cudaMemcpyDeviceToHost), "read unique");
    if (pos && TK) CUDA_TRY(cudaMemcpy(pos, p.pos, TK * 4, cudaMemcpyDeviceToHost), "read pos");
    if (tok && TK) CUDA_TRY(cudaMemcpy(tok, p.tok, TK * 4, cudaMemcpyDeviceToHost), "read tok");
    return COLI_OK;
}

COLI_API coli_status coli_moe_set_profiling(coli_moe_layer* L, int enable) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    DeviceGuard guard(L->device);
    if (enable && !L->ev[0][0]) {
        for (auto& set : L->ev)
            for (auto& e : set) CUDA_TRY(cudaEventCreate(&e), "cudaEventCreate");
    }
    if (L->ev[0][0]) CUDA_TRY(cudaDeviceSynchronize(), "sync");
    L->profiling = enable != 0;
    L->prof_next = 0;
    L->prof_issued = L->prof_folded = 0;
    for (double& t : L->prof_total) t = 0.0;
    return COLI_OK;
}

COLI_API coli_status coli_moe_get_profile(coli_moe_layer* L, double* stage_ms_total, int64_t* n_forwards) {
    if (!L || !stage_ms_total) return fail(COLI_EINVAL, "NULL argument");
    DeviceGuard guard(L->device);
    const int K = coli_moe_layer::kRing;
    while (L->prof_folded < L->prof_issued) {
        const int64_t pending = L->prof_issued - L->prof_folded;   // <= K
        const int r = (int)(((L->prof_next - pending) % K + K) % K);  // oldest pending slot
        CUDA_TRY(prof_fold(L, r), "profile");
    }
    for (int i = 0; i < COLI_N_STAGES; ++i) stage_ms_total[i] = L->prof_total[i];
    if (n_forwards) *n_forwards = L->prof_folded;
    return COLI_OK;
}

COLI_API const char* coli_moe_stage_name(int stage) {
    static const char* names[COLI_N_STAGES] = {"router", "topk", "plan", "gateup", "down", "combine", "fused", "cache"};
    return (stage >= 0 && stage < COLI_N_STAGES) ? names[stage] : "";
}

COLI_API coli_status coli_moe_cache_stats(coli_moe_layer* L, coli_cache_stats* stats, int64_t* usage, int reset) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!L->cached) return fail(COLI_EINVAL, "not a cached layer");
    DeviceGuard guard(L->device);
    CUDA_TRY(cudaStreamSynchronize(L->copy_stream), "wait for prefetch copies");
    if (stats) {
        stats->hits = L->cache.hits;
        stats->misses = L->cache.misses;
        stats->bytes_h2d = L->bytes_h2d;
        stats->prefetched = L->n_prefetched;
        stats->prefetch_used = L->prefetch_used;
        stats->predicted = L->predicted;
        stats->predicted_of = L->predicted_of;
        stats->resident_slots = L->cache.slots;
        int np = 0;
        for (int e = 0; e < L->d.E; ++e) np += L->cache.is_pinned(e);
        stats->n_pinned = np;
    }
    if (usage)
        for (int e = 0; e < L->d.E; ++e) usage[e] = L->cache.uses[e];
    if (reset) {
        L->cache.hits = L->cache.misses = 0;
        L->bytes_h2d = L->n_prefetched = L->prefetch_used = L->predicted = L->predicted_of = 0;
    }
    return COLI_OK;
}

COLI_API coli_status coli_moe_cache_pin(coli_moe_layer* L, const int32_t* ids, int n) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!L->cached) return fail(COLI_EINVAL, "not a cached layer");
    if (n < 0 || (n > 0 && !ids)) return fail(COLI_EINVAL, "bad id list");
    const int reserve = (int)std::min<int64_t>((int64_t)L->cfg.max_tokens * L->d.K, L->d.E);
    if (!L->cache.pin(ids, n, reserve))
        return fail(COLI_EINVAL, "ids out of range, or more than resident_slots - min(n_experts, max_tokens * top_k)");
    DeviceGuard guard(L->device);
    coli_status st = cache_prefetch(L, ids, n);  // pinned experts are never the victims, so all of them fit
    if (st != COLI_OK) return st;
    CUDA_TRY(cudaStreamSynchronize(L->copy_stream), "pin copies");
    return COLI_OK;
}

COLI_API coli_status coli_moe_cache_prefetch(coli_moe_layer* L, const int32_t* ids, int n) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!L->cached) return fail(COLI_EINVAL, "not a cached layer");
    if (n < 0 || (n > 0 && !ids)) return fail(COLI_EINVAL, "bad id list");
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= L->d.E) return fail(COLI_EINVAL, "expert id out of range");
    DeviceGuard guard(L->device);
    return cache_prefetch(L, ids, n);
}

COLI_API coli_status coli_moe_cache_slots(const coli_moe_layer* L, int32_t* slots) {
    if (!L || !slots) return fail(COLI_EINVAL, "NULL argument");
    if (!L->cached) return fail(COLI_EINVAL, "not a cached layer");
    for (int e = 0; e < L->d.E; ++e) slots[e] = L->cache.slot(e);
    return COLI_OK;
}

COLI_API coli_status coli_moe_cache_set_lookahead(coli_moe_layer* L, int enable) {
    if (!L) return fail(COLI_EINVAL, "layer is NULL");
    if (!L->cached) return fail(COLI_EINVAL, "not a cached layer");
    if (enable < 0 || enable > 1) return fail(COLI_EINVAL, "enable must be 0 or 1");
    L->lookahead = enable != 0;
    if (!L->lookahead) L->ahead_valid = false;
    return COLI_OK;
}

COLI_API const char* coli_status_string(coli_status s) {
    switch (s) {
        case COLI_OK: return "ok";
        case COLI_EINVAL: return "invalid argument";
        case COLI_ENOMEM: return "out of memory";
        case COLI_ECUDA: return "CUDA error";
        case COLI_EUNSUPPORTED: return "unsupported";
    }
    return "unknown status";
}

COLI_API const char* coli_last_error(void) { return g_last_error.c_str(); }

namespace coli {
void set_last_error(const std::string& what) { g_last_error = what; }
}  // namespace coli
