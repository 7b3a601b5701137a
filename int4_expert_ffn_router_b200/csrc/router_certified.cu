// router_certified.cu -- the router of token batches on the integer tensor
// cores, with a certified selection and fp64 only where the certificate fails.
//
// The router and its top-K are those of router.cu (logits Wr x + b, the K
// largest, equal logits to the lower id, softmax over the K): "Colibri: 2400
// lines of pure C ..." (kechuai.cn), section 一. An fp64 GEMM of a 2048-token
// batch is bound by the FP64 rate; this form computes every logit exactly up
// to a tiny, rigorously bounded representation error:
//
//   x_t ~ xh_t = 2^s_t * qx_t,  qx_t integers, |qx| < 2^30 (per-token scale)
//   Wr_e ~ wh_e = 2^r_e * qw_e,  qw_e integers, |qw| < 2^30 (per-expert scale)
//   each q as four signed base-256 digits d_0 .. d_3 (d_0 most significant):
//     q = d_0 2^24 + d_1 2^16 + d_2 2^8 + d_3,  every d in [-128, 127]
//
// One int8 tensor-core GEMM (tcgen05.mma kind::i8, exact int32 accumulation)
// forms all 16 digit products P_pq = sum_h dw_p[h] dx_q[h] of a (token,
// expert) pair; sum_pq 2^(8(6-p-q)) P_pq = qw . qx exactly, and
//   v = 2^(s+r) (qw . qx) + b   (fp64, three additions and the bias rounded)
// differs from the exact logit by at most
//   eps = ||Wr_e - wh_e|| ||x_t|| + ||wh_e|| ||x_t - xh_t||
//         + 7u max|Wr_e| sqrt(H) ||xh_t|| + 2u |v|,   u = 2^-53
// (norms in fp64, rounded up). The scales keep the largest element of a row
// in [2^29, 2^30), so fp32 and bf16 values at most 2^6 below a row's largest
// are represented exactly; eps is about 1e-9 of ||Wr_e|| ||x_t||. A token is
// certified when its K selected intervals [v - eps, v + eps] lie strictly
// above every other expert's and strictly ordered among themselves, and the
// weights' error bound (at most 2.01 max eps relative) stays below 5e-7
// (with top-p, no running sum within that bound of p). Then the ids and their
// order are those of the exact logits, and of any fp64 evaluation that does
// not itself hit such a tie; the weights come from v. Any other token gets all
// of its logits in fp64 and the fp64 top-K, as router.cu computes them.
#include <cuda.h>

#include <cfloat>
#include <cstring>

#include "common.cuh"
#include "kernels.cuh"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace coli {
namespace {

// GEMM tile: 32 experts x 4 digit planes = 128 rows of A (the MMA's M) and
// tb tokens x 4 digit planes = 4 tb rows of B (its N; tb <= 64, a multiple of
// 8, chosen per call so that the SMs' loads are even); 128 inputs (bytes) of
// the input dimension per pipeline stage, four K = 32 MMAs each.
constexpr int kRxE = 32, kRxT = 64, kRxK = 128;
constexpr int kRxTiles[5] = {64, 56, 48, 40, 32};  // token rows per tile the launcher chooses from
constexpr int kRxM = 4 * kRxE, kRxN = 4 * kRxT;
constexpr int kRxStages = 2;
constexpr int kRxABytes = kRxM * kRxK;                 // 16 KB
constexpr int kRxBBytes = kRxN * kRxK;                 // 32 KB for the largest tile (64 tokens)
constexpr int kRxStageBytes = kRxABytes + kRxBBytes;   // 48 KB: the stride of a stage
constexpr int kRxStageOut = 4 * kRxT * kRxE * 8;       // epilogue: the four digit-plane terms, fp64
static_assert(kRxStageOut <= kRxStages * kRxStageBytes, "the epilogue reuses the pipeline buffers");
constexpr int kRxOffBar = kRxStages * kRxStageBytes;
constexpr int kRxSmem = kRxOffBar + 64 + 1024;         // barriers, tensor-memory slot, flag, alignment slack
constexpr int kRxThreads = 192;                        // producer, MMA, four epilogue warps
constexpr uint32_t kRxTmemCols = 256;
constexpr uint64_t kRxWaitNs = 1000000000ull;          // every wait gives up after 1 s (default)

// Error-bound constants (u = 2^-53): the three fp64 additions of the digit
// terms, at most 3.01u of sum |term| <= 2.02 max|Wr_e| sqrt(H) ||xh_t||, with
// margin; the bias addition; the norms' own rounding (fp64 sums of at most
// 2^16 squares).
constexpr double kRxAddBound = 7.0 * 1.1102230246251565e-16;
constexpr double kRxBiasBound = 2.3e-16;
constexpr double kRxNormUp = 1.0 + 1e-10;
constexpr double kRxWeightTol = 5e-7;

template <typename XT>
__device__ __forceinline__ void rx_load8(const XT* p, float v[8]);
template <>
__device__ __forceinline__ void rx_load8<float>(const float* p, float v[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void rx_load8<__nv_bfloat16>(const __nv_bfloat16* p, float v[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// The four signed base-256 digits of q (|q| < 2^30) as the bytes of one word,
// byte k the digit of weight 2^8k: adding 128 at each of the three low digit
// positions makes every low digit d + 128 an ordinary byte (0..255) and leaves
// the top digit in the arithmetic top byte; xor 0x80 takes 128 off again.
__device__ __forceinline__ uint32_t rx_digits(int q) { return (uint32_t)(q + 0x808080) ^ 0x808080u; }

// Byte transpose of four digit words (elements 0..3) into four plane words:
// plane word k holds byte k of each element, element i in byte i.
__device__ __forceinline__ void rx_planes4(const uint32_t w[4], uint32_t out[4]) {
    const uint32_t lo01 = __byte_perm(w[0], w[1], 0x5140), lo23 = __byte_perm(w[2], w[3], 0x5140);
    const uint32_t hi01 = __byte_perm(w[0], w[1], 0x7362), hi23 = __byte_perm(w[2], w[3], 0x7362);
    out[0] = __byte_perm(lo01, lo23, 0x5410);
    out[1] = __byte_perm(lo01, lo23, 0x7632);
    out[2] = __byte_perm(hi01, hi23, 0x5410);
    out[3] = __byte_perm(hi01, hi23, 0x7632);
}

// Block-wide fp64 sums over 256 threads; `red` holds 8 x 4 doubles.
__device__ __forceinline__ void rx_block_sum3(double& a, double& b, double& c, double* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    __syncthreads();
    if (lane == 0) { red[4 * warp] = a; red[4 * warp + 1] = b; red[4 * warp + 2] = c; }
    __syncthreads();
    a = b = c = 0.0;
    for (int w = 0; w < 8; ++w) { a += red[4 * w]; b += red[4 * w + 1]; c += red[4 * w + 2]; }
}

// One CTA (256 threads) per row of n values (n % 8 == 0): the power-of-two
// scale 2^s that puts the row's largest magnitude in [2^29, 2^30), the four
// digit planes of the row scaled by 2^-s and rounded to integers (plane p at
// out + p * plane), and the norms ||v||, ||v - vh||, ||vh|| rounded up. A row
// holding a non-finite value gets a NaN norm (its logits then fail every
// certificate) and zero digits.
template <typename XT>
__device__ __forceinline__ void rx_split_row(const XT* __restrict__ row, int n, uint8_t* __restrict__ out,
                                             size_t plane, int* scale, double* nv, double* nd, double* nq,
                                             float* vmax) {
    __shared__ unsigned smax;
    __shared__ int sbad;
    __shared__ double red[32];
    if (threadIdx.x == 0) { smax = 0u; sbad = 0; }
    __syncthreads();
    float m = 0.0f;
    bool bad = false;
    for (int h = 8 * threadIdx.x; h < n; h += 8 * blockDim.x) {
        float v[8];
        rx_load8<XT>(row + h, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float a = fabsf(v[i]);
            bad |= !(a <= FLT_MAX);
            m = fmaxf(m, a);
        }
    }
    atomicMax(&smax, __float_as_uint(m));
    if (bad) sbad = 1;
    __syncthreads();
    const float amax = __uint_as_float(smax);
    const bool any_bad = sbad != 0;
    int ex = 0;
    if (amax > 0.0f && !any_bad) frexpf(amax, &ex);  // amax = f 2^ex, f in [0.5, 1)
    const int s = (amax > 0.0f && !any_bad) ? ex - 30 : 0;
    // y = v 2^-s exactly (fp64; s in [-180, 130]), q = rint(y), y - q exact:
    // ||v - vh||^2 = 2^2s sum (y - q)^2, ||vh||^2 = 2^2s sum q^2
    const double down = __longlong_as_double((long long)(1023 - s) << 52);
    double sv = 0.0, sd = 0.0, sq = 0.0;
    for (int h = 8 * threadIdx.x; h < n; h += 8 * blockDim.x) {
        float v[8];
        rx_load8<XT>(row + h, v);
        uint32_t wd[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double xv = (double)v[i];
            const double y = any_bad ? 0.0 : xv * down;
            const double yr = rint(y);
            const double res = y - yr;
            sv = fma(xv, xv, sv);
            sd = fma(res, res, sd);
            sq = fma(yr, yr, sq);
            wd[i] = rx_digits((int)yr);
        }
        uint32_t pa[4], pb[4];  // plane words of elements 0..3 and 4..7; byte 3 is digit d_0 (plane 0)
        rx_planes4(wd, pa);
        rx_planes4(wd + 4, pb);
#pragma unroll
        for (int p = 0; p < 4; ++p)
            *reinterpret_cast<uint2*>(out + (size_t)p * plane + h) = make_uint2(pa[3 - p], pb[3 - p]);
    }
    const double up2 = __longlong_as_double((long long)(1023 + 2 * s) << 52);
    sd *= up2;
    sq *= up2;
    rx_block_sum3(sv, sd, sq, red);
    if (threadIdx.x == 0) {
        *scale = s;
        *nv = any_bad ? __longlong_as_double(0x7ff8000000000000ll) : sqrt(sv) * kRxNormUp;
        *nd = sqrt(sd) * kRxNormUp;
        *nq = sqrt(sq) * kRxNormUp;
        if (vmax) *vmax = amax;
    }
}

// Digit planes of the router rows (once, when the weights are loaded):
// wd8 [4][E][H], scale r_e, and the per-expert bound factors
// wb[e] = {||Wr_e - wh_e||, ||wh_e||, 7u max|Wr_e| sqrt(H)}.
__global__ void __launch_bounds__(256) router_split_w_kernel(const float* __restrict__ wr, int E, int H,
                                                             uint8_t* __restrict__ wd8, int* __restrict__ wscale,
                                                             double* __restrict__ wb) {
    const int e = blockIdx.x;
    __shared__ float wmax;
    double nv;
    rx_split_row<float>(wr + (size_t)e * H, H, wd8 + (size_t)e * H, (size_t)E * H, wscale + e, &nv, wb + 3 * e,
                        wb + 3 * e + 1, &wmax);
    __syncthreads();
    if (threadIdx.x == 0) {
        // wb[3e] was ||Wr_e - wh_e||; a non-finite row makes every bound NaN
        if (nv != nv) wb[3 * e] = nv;
        wb[3 * e + 2] = kRxAddBound * (double)wmax * sqrt((double)H) * kRxNormUp;
    }
}

// Digit planes of a token batch: xd8 [4][Tm][H] (plane stride Tm * H), scale
// s_t, and xb[t] = {||x_t||, ||x_t - xh_t||, ||xh_t||}. CTA 0 also clears the
// fallback count of this call.
template <typename XT>
__global__ void __launch_bounds__(256) router_split_x_kernel(const XT* __restrict__ x, int T, int H, int Tm,
                                                             uint8_t* __restrict__ xd8, int* __restrict__ xscale,
                                                             double* __restrict__ xb, int* __restrict__ fail) {
    const int t = blockIdx.x;
    if (t == 0 && threadIdx.x == 0) *fail = 0;
    rx_split_row<XT>(x + (size_t)t * H, H, xd8 + (size_t)t * H, (size_t)Tm * H, xscale + t, xb + 3 * t,
                     xb + 3 * t + 1, xb + 3 * t + 2, nullptr);
}

// TMA tile load of box (x, y, z) of a 3D tensor map (no multicast).
__device__ __forceinline__ void rx_tma_3d(uint32_t dst, const void* tmap, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

// Four MMAs (K = 32 each, one 128-byte stage row) of int8 digits into the
// int32 accumulator, then one commit to `bar`. Warp-converged: one elected
// lane issues.
__device__ __forceinline__ void rx_mma4_commit(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate,
                                               uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e, p, t;\n\t.reg .b64 a1, a2, a3, b1, b2, b3;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %4, 0;\n\tsetp.eq.b32 t, %4, %4;\n\t"
        "add.s64 a1, %1, 2;\n\tadd.s64 a2, %1, 4;\n\tadd.s64 a3, %1, 6;\n\t"
        "add.s64 b1, %2, 2;\n\tadd.s64 b2, %2, 4;\n\tadd.s64 b3, %2, 6;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], a1, b1, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], a2, b2, %3, t;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::i8 [%0], a3, b3, %3, t;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%5];\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(bar)
        : "memory");
}

// Instruction descriptor of kind::i8: D s32 (bits 4-5 = 2), A and B signed
// 8-bit (bits 7-9, 10-12 = 1), both K-major, N / 8 at bit 17, M / 16 at bit 24.
__host__ __device__ constexpr uint32_t rx_idesc_s8(int m, int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ bool rx_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err, int site,
                                        uint64_t limit) {
    if (mbar_try_wait_sleep(bar, parity, 200000)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 200000)) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > limit) {
            *abort_flag = 1;
            atomicCAS(err, 0, site);
            return false;
        }
    }
}
__device__ __forceinline__ bool rx_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* err,
                                             int site, uint64_t limit) {
    const bool ok = rx_wait(bar, parity, abort_flag, err, site, limit);
    return __all_sync(0xffffffffu, ok);
}

struct __align__(64) RxArgs {
    CUtensorMap wmap;  // digit planes of the router rows: dims (H, E, 4), box (128, 32, 1)
    CUtensorMap xmap;  // digit planes of the batch: dims (H, Tm, 4), box (128, tb, 1)
    const int* wscale;
    const int* xscale;
    const float* bias;
    double* logits;    // [T][E]
    int T, H, E;
    int tb;            // token rows per tile
    int* err;
    uint64_t wait_ns;  // bound of every wait
    int wait_test;     // testing aid: the MMA warp first waits on a barrier that nothing completes
};

// CTA (bx, by): experts 32 bx .. +31, tokens tb by .. +tb-1. Warp 0 (one lane)
// loads each stage's 4 + 4 digit boxes with TMA; warp 1 allocates the
// accumulator (128 lanes x 4 tb int32 columns: lane 32 p + e, column tb q + t)
// and issues the MMAs; warps 2..5 (lane quarter p = warp % 4) read it back:
// term_p(t, e) = 2^(8(3-p)) sum_q 2^(8(3-q)) P_pq, exact in fp64 (below
// 2^53), staged in shared memory, then v = ((term_0 + term_1) + term_2) +
// term_3 scaled by 2^(s_t + r_e), plus the bias.
__global__ void __launch_bounds__(kRxThreads, 1) router_i8_kernel(const __grid_constant__ RxArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + kRxOffBar);  // [kRxStages]
    uint64_t* empty = full + kRxStages;                              // [kRxStages]
    uint64_t* accfull = empty + kRxStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accfull + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tb = a.tb;
    const int e0 = blockIdx.x * kRxE, t0 = blockIdx.y * tb;
    const uint32_t stage_tx = kRxABytes + 4 * tb * kRxK;  // bytes one stage's boxes bring
    const int nkb = (a.H + kRxK - 1) / kRxK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRxStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accfull, 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) {
        tc_alloc(tmem_slot, kRxTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0) {
        if (lane == 0) {
            int kb = 0;
            for (; kb < nkb; ++kb) {
                const int s = kb % kRxStages;
                if (!rx_wait(&empty[s], ((kb / kRxStages) & 1) ^ 1, abort_flag, a.err, 41, a.wait_ns)) break;
                uint8_t* st = sm + s * kRxStageBytes;
                mbar_arrive_expect_tx(&full[s], stage_tx);
#pragma unroll
                for (int p = 0; p < 4; ++p)
                    rx_tma_3d(smem_addr(st + p * (kRxE * kRxK)), &a.wmap, kb * kRxK, e0, p, &full[s]);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    rx_tma_3d(smem_addr(st + kRxABytes + q * (tb * kRxK)), &a.xmap, kb * kRxK, t0, q, &full[s]);
            }
            // copies still in flight (after an abort) land before the CTA exits
            const int first = kb > kRxStages ? kb - kRxStages : 0;
            const uint64_t tw = globaltimer_ns();
            for (int k = first; k < kb; ++k)
                while (!mbar_try_wait(&full[k % kRxStages], (k / kRxStages) & 1) && globaltimer_ns() - tw < a.wait_ns) {
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        const uint32_t idesc = rx_idesc_s8(kRxM, 4 * tb);
        const uint64_t adesc0 = tc_sdesc_sw128(smem_addr(sm));
        bool issued = false;
        // testing aid: accfull completes only after this warp's own commit, so the launch gives up
        if (a.wait_test) ok = rx_wait_warp(accfull, 0, abort_flag, a.err, 44, a.wait_ns);
        for (int kb = 0; ok && kb < nkb; ++kb) {
            const int s = kb % kRxStages;
            if (!rx_wait_warp(&full[s], (kb / kRxStages) & 1, abort_flag, a.err, 42, a.wait_ns)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = adesc0 + (uint64_t)((s * kRxStageBytes) >> 4);
            const uint64_t bd = ad + (uint64_t)(kRxABytes >> 4);
            rx_mma4_commit(tmem, ad, bd, idesc, kb != 0, smem_addr(&empty[s]));
            issued = true;
        }
        if (issued) {
            // accfull completes when every MMA issued above has completed (also after an abort,
            // so the tensor memory is never released under a running MMA)
            tc_commit_elect(accfull);
            const uint64_t tw = globaltimer_ns();
            while (!mbar_try_wait(accfull, 0) && globaltimer_ns() - tw < a.wait_ns) {
            }
        }
        __syncwarp();
    } else {
        const int p = warp & 3;
        double* stage = reinterpret_cast<double*>(sm);  // [4][kRxT][kRxE]
        ok = rx_wait_warp(accfull, 0, abort_flag, a.err, 43, a.wait_ns) && !*abort_flag;
        if (ok) {
            tc_fence_after();
            const uint32_t tl = tmem + ((uint32_t)(32 * p) << 16);
            const double wp = p == 0 ? 16777216.0 : p == 1 ? 65536.0 : p == 2 ? 256.0 : 1.0;
#pragma unroll 1
            // chunks of 16 columns per plane; a last chunk that runs past the plane's tb
            // columns reads columns that are skipped (all inside the 256 allocated)
            for (int c = 0; 16 * c < tb; ++c) {
                uint32_t v0[16], v1[16], v2[16], v3[16];
                tc_ld16_wait(tl + 0 * tb + 16 * c, v0);
                tc_ld16_wait(tl + 1 * tb + 16 * c, v1);
                tc_ld16_wait(tl + 2 * tb + 16 * c, v2);
                tc_ld16_wait(tl + 3 * tb + 16 * c, v3);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (16 * c + i >= tb) break;
                    const long long sp = ((long long)(int)v0[i] << 24) + ((long long)(int)v1[i] << 16) +
                                         ((long long)(int)v2[i] << 8) + (long long)(int)v3[i];
                    stage[((size_t)p * kRxT + 16 * c + i) * kRxE + lane] = (double)sp * wp;
                }
            }
        }
        // the four epilogue warps (128 threads) meet; the pipeline buffers now hold the terms
        named_bar(1, 128);
        const bool all_ok = ok && !*abort_flag;
        if (all_ok) {
            const int e = e0 + lane;
            const bool ein = e < a.E;
            const int r = ein ? __ldg(a.wscale + e) : 0;
            const double b = ein ? (double)__ldg(a.bias + e) : 0.0;
            for (int tt = warp - 2; tt < tb; tt += 4) {
                const int t = t0 + tt;
                if (t >= a.T || !ein) continue;
                const double v = ((stage[(0 * kRxT + tt) * kRxE + lane] + stage[(1 * kRxT + tt) * kRxE + lane]) +
                                  stage[(2 * kRxT + tt) * kRxE + lane]) +
                                 stage[(3 * kRxT + tt) * kRxE + lane];
                a.logits[(size_t)t * a.E + e] = ldexp(v, __ldg(a.xscale + t) + r) + b;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tc_dealloc(tmem, kRxTmemCols);
}

// One warp per token: the bound of each logit, the K largest (descending,
// equal values to the lower id), the certificate, then either the ids and
// weights (adaptive top-p included) or the token on the fallback list.
__global__ void __launch_bounds__(256) router_certify_kernel(const double* __restrict__ logits,
                                                             const double* __restrict__ wb,
                                                             const double* __restrict__ xb, int T, int E, int K,
                                                             double topp, int e_lo, int e_hi,
                                                             int32_t* __restrict__ ids, float* __restrict__ w,
                                                             int* __restrict__ fail) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= T) return;
    const double xn = xb[3 * t], xd = xb[3 * t + 1], xq = xb[3 * t + 2];
    auto bound = [&](int e, double v) {
        return (wb[3 * e] * xn + wb[3 * e + 1] * xd + wb[3 * e + 2] * xq) * (1.0 + 1e-9) + kRxBiasBound * fabs(v) +
               1e-300;
    };
    // this lane's experts lane + 32 i (i < 8): key and interval
    unsigned long long ks[8];
    int is[8];
    double lo8[8], hi8[8];
    bool present[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        present[i] = e < E;
        ks[i] = 0ull;
        is[i] = 0x7fffffff;
        lo8[i] = hi8[i] = 0.0;
        if (present[i]) {
            const double v = logits[(size_t)t * E + e];
            const double eps = bound(e, v);
            ks[i] = order_key(v);
            is[i] = e;
            lo8[i] = v - eps;
            hi8[i] = v + eps;
        }
    }
    // the K largest: each lane sorts its 8 entries, then K rounds take the warp's best head
    cx8(ks, is, 0, 1); cx8(ks, is, 2, 3); cx8(ks, is, 4, 5); cx8(ks, is, 6, 7);
    cx8(ks, is, 0, 2); cx8(ks, is, 1, 3); cx8(ks, is, 4, 6); cx8(ks, is, 5, 7);
    cx8(ks, is, 1, 2); cx8(ks, is, 5, 6);
    cx8(ks, is, 0, 4); cx8(ks, is, 1, 5); cx8(ks, is, 2, 6); cx8(ks, is, 3, 7);
    cx8(ks, is, 2, 4); cx8(ks, is, 3, 5);
    cx8(ks, is, 1, 2); cx8(ks, is, 3, 4); cx8(ks, is, 5, 6);
    int my_id = -1;
    unsigned long long my_key = 0ull, top_key = 0ull;
    unsigned selmask = 0u;  // this lane's selected entries (expert lane + 32 i: bit i)
    for (int r = 0; r < K; ++r) {
        const unsigned khi = (unsigned)(ks[0] >> 32), klo = (unsigned)ks[0];
        const unsigned bhi = __reduce_max_sync(0xffffffffu, khi);
        const unsigned blo = __reduce_max_sync(0xffffffffu, khi == bhi ? klo : 0u);
        const bool holds = khi == bhi && klo == blo;
        const int bi = (int)__reduce_min_sync(0xffffffffu, holds ? (unsigned)is[0] : 0x7fffffffu);
        if (holds && is[0] == bi) {
            selmask |= 1u << ((bi - lane) >> 5);
#pragma unroll
            for (int i = 0; i < 7; ++i) { ks[i] = ks[i + 1]; is[i] = is[i + 1]; }
            ks[7] = 0ull;
            is[7] = 0x7fffffff;
        }
        const unsigned long long bk = ((unsigned long long)bhi << 32) | blo;
        if (r == 0) top_key = bk;
        if (lane == r) { my_id = bi; my_key = bk; }
    }
    // certificate 1: every selected interval above every other one
    double sel_lo = 1e300, oth_hi = -1e300;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (!present[i]) continue;
        if ((selmask >> i) & 1u) sel_lo = fmin(sel_lo, lo8[i]);
        else oth_hi = fmax(oth_hi, hi8[i]);
    }
    // certificate 2: the selected intervals strictly ordered; the largest bound among them
    const bool mine = lane < K && my_id >= 0 && my_id < E;
    const double my_v = mine ? key_value(my_key) : 0.0;
    const double my_eps = mine ? bound(my_id, my_v) : 0.0;
    const double next_hi = __shfl_down_sync(0xffffffffu, my_v + my_eps, 1);
    bool ok = lane >= K - 1 || (mine && my_v - my_eps > next_hi);
    double m = my_eps;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sel_lo = fmin(sel_lo, __shfl_xor_sync(0xffffffffu, sel_lo, o));
        oth_hi = fmax(oth_hi, __shfl_xor_sync(0xffffffffu, oth_hi, o));
        m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    }
    // certificate 3: the weights' error bound (relative 2.01 m), and with top-p no running
    // sum of the weights within that bound of p
    ok = __all_sync(0xffffffffu, ok) && sel_lo > oth_hi && 2.01 * m <= kRxWeightTol;
    if (ok && topp > 0.0 && topp < 1.0) {
        const double ex = lane < K ? exp(my_v - key_value(top_key)) : 0.0;
        double z = ex;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        const double wk = ex / z;
        double cum = 0.0;
        for (int j = 0; j < K; ++j) {
            cum += __shfl_sync(0xffffffffu, wk, j);
            ok = ok && fabs(cum - topp) > 2.01 * m + 1e-12;
        }
    }
    if (!ok) {
        if (lane == 0) fail[1 + atomicAdd(fail, 1)] = t;
        return;
    }
    int id;
    float wt;
    topk_weights(lane < K ? my_key : 0ull, top_key, lane < K ? my_id : -1, K, topp, lane, &id, &wt);
    if (lane < K) {
        ids[(size_t)t * K + lane] = (id >= e_lo && id < e_hi) ? id : -1;
        w[(size_t)t * K + lane] = wt;
    }
}

// Fallback: fp64 logits of the listed tokens. CTA (bx, by): experts 2bx,
// 2bx+1 (four warps each, a quarter of H per warp) for listed tokens by,
// by + gridDim.y, ...
template <typename XT>
__global__ void __launch_bounds__(256) router_fallback_kernel(const float* __restrict__ wr, const float* __restrict__ bias,
                                                              const XT* __restrict__ x, int H, int E,
                                                              const int* __restrict__ fail, double* __restrict__ logits) {
    __shared__ double part[8];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 2 + (warp >> 2), quarter = warp & 3, seg = H / 4;
    const int n = *fail;
    for (int f = blockIdx.y; f < n; f += gridDim.y) {
        const int t = fail[1 + f];
        double s = 0.0;
        if (e < E) {
            const float* wrow = wr + (size_t)e * H + quarter * seg;
            const XT* xrow = x + (size_t)t * H + quarter * seg;
            for (int h = lane; h < seg; h += 32) {
                float v;
                if constexpr (sizeof(XT) == 4) v = xrow[h];
                else v = __bfloat162float(xrow[h]);
                s = fma((double)wrow[h], (double)v, s);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[warp] = s;
        __syncthreads();
        if (threadIdx.x < 2) {
            const int ee = blockIdx.x * 2 + threadIdx.x;
            if (ee < E) {
                const double* p = part + 4 * threadIdx.x;
                logits[(size_t)t * E + ee] = ((p[0] + p[1]) + p[2]) + p[3] + (double)bias[ee];
            }
        }
        __syncthreads();
    }
}

// Fallback top-K of the listed tokens, one warp per token.
__global__ void __launch_bounds__(256) router_fallback_topk_kernel(const double* __restrict__ logits, int E, int K,
                                                                   double topp, int e_lo, int e_hi,
                                                                   const int* __restrict__ fail,
                                                                   int32_t* __restrict__ ids, float* __restrict__ w) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = *fail;
    for (int f = blockIdx.x * 8 + warp; f < n; f += gridDim.x * 8) {
        const int t = fail[1 + f];
        int id;
        float wt;
        warp_topk8<true>(logits + (size_t)t * E, E, K, topp, lane, &id, &wt);
        if (lane < K) {
            ids[(size_t)t * K + lane] = (id >= e_lo && id < e_hi) ? id : -1;
            w[(size_t)t * K + lane] = wt;
        }
    }
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// 3D int8 map over four digit planes of rows x H bytes (plane stride rows *
// H): box 128 bytes x box_rows rows x 1 plane, 128-byte swizzle, zero fill
// outside the tensor.
cudaError_t rx_encode(void* map, const uint8_t* base, int rows, int H, int box_rows) {
    static EncodeFn encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        encode = reinterpret_cast<EncodeFn>(fn);
    }
    if (((uintptr_t)base & 15u) || H % 16 || rows < 1) return cudaErrorInvalidValue;
    const cuuint64_t dims[3] = {(cuuint64_t)H, (cuuint64_t)rows, 4};
    const cuuint64_t strides[2] = {(cuuint64_t)H, (cuuint64_t)rows * H};
    const cuuint32_t box[3] = {(cuuint32_t)kRxK, (cuuint32_t)box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = encode(reinterpret_cast<CUtensorMap*>(map), CU_TENSOR_MAP_DATA_TYPE_UINT8, 3,
                              const_cast<uint8_t*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace

bool router_certified_supported(int H, int E) { return H % 16 == 0 && H >= kRxK && H <= 65536 && E >= 1 && E <= 256; }

size_t router_certified_smem_bytes() { return kRxSmem; }

cudaError_t router_certified_prepare(RouterCert& rc, const float* wr, cudaStream_t st) {
    if (!router_certified_supported(rc.H, rc.E) || rc.Tm < 1) return cudaErrorInvalidValue;
    router_split_w_kernel<<<rc.E, 256, 0, st>>>(wr, rc.E, rc.H, rc.wd8, rc.wscale, rc.wb);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((e = rx_encode(rc.maps, rc.wd8, rc.E, rc.H, kRxE)) != cudaSuccess) return e;
    for (int i = 0; i < 5; ++i)
        if ((e = rx_encode(rc.maps + (1 + i) * sizeof(CUtensorMap), rc.xd8, rc.Tm, rc.H, kRxTiles[i])) != cudaSuccess)
            return e;
    return cudaFuncSetAttribute(router_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRxSmem);
}

cudaError_t launch_router_certified(const RouterCert& rc, const float* wr, const float* bias, const void* x,
                                    coli_dtype dt, int T, int K, double topp, int e_lo, int e_hi, double* logits,
                                    int32_t* ids, float* w, int* err, int64_t wait_ns, int wait_test,
                                    cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (T > rc.Tm || K < 1 || K > 32) return cudaErrorInvalidValue;
    if (e_hi < 0) e_hi = rc.E;
    const int H = rc.H, E = rc.E;
    if (dt == COLI_F32)
        router_split_x_kernel<float><<<T, 256, 0, st>>>((const float*)x, T, H, rc.Tm, rc.xd8, rc.xscale, rc.xb, rc.fail);
    else
        router_split_x_kernel<__nv_bfloat16><<<T, 256, 0, st>>>((const __nv_bfloat16*)x, T, H, rc.Tm, rc.xd8,
                                                                rc.xscale, rc.xb, rc.fail);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    RxArgs a;
    memcpy(&a.wmap, rc.maps, sizeof(CUtensorMap));
    // the tile height whose busiest SM has the least work: tiles per SM (2 resident) x rows per tile
    int pick = 0;
    long best = -1;
    for (int i = 0; i < 5; ++i) {
        const long tiles = (long)((E + kRxE - 1) / kRxE) * ((T + kRxTiles[i] - 1) / kRxTiles[i]);
        const long load = ((tiles + rc.n_sm - 1) / rc.n_sm) * kRxTiles[i];
        if (best < 0 || load < best) { best = load; pick = i; }
    }
    a.tb = kRxTiles[pick];
    memcpy(&a.xmap, rc.maps + (1 + pick) * sizeof(CUtensorMap), sizeof(CUtensorMap));
    a.wscale = rc.wscale;
    a.xscale = rc.xscale;
    a.bias = bias;
    a.logits = logits;
    a.T = T;
    a.H = H;
    a.E = E;
    a.err = err;
    a.wait_ns = wait_ns > 0 ? (uint64_t)wait_ns : kRxWaitNs;
    a.wait_test = wait_test;
    const dim3 g((E + kRxE - 1) / kRxE, (T + a.tb - 1) / a.tb);
    router_i8_kernel<<<g, kRxThreads, kRxSmem, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    router_certify_kernel<<<(T + 7) / 8, 256, 0, st>>>(logits, rc.wb, rc.xb, T, E, K, topp, e_lo, e_hi, ids, w,
                                                       rc.fail);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 gf((E + 1) / 2, 4);
    if (dt == COLI_F32) router_fallback_kernel<float><<<gf, 256, 0, st>>>(wr, bias, (const float*)x, H, E, rc.fail, logits);
    else router_fallback_kernel<__nv_bfloat16><<<gf, 256, 0, st>>>(wr, bias, (const __nv_bfloat16*)x, H, E, rc.fail, logits);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    router_fallback_topk_kernel<<<16, 256, 0, st>>>(logits, E, K, topp, e_lo, e_hi, rc.fail, ids, w);
    return cudaGetLastError();
}

}  // namespace coli
