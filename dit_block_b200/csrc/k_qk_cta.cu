// k_qk_cta.cu -- QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合"]
// (bf16, head_dim 128, q and k both given) with one CTA per token whose q row and k row
// land in shared memory by two bulk asynchronous copies.
//
// Why: the op is an in-place stream of 4 bytes per element with little arithmetic, so it is
// bound by the bytes each SM keeps in flight.  Rows held in registers cap that at what the
// register file spares (a persistent warp per row, k_qk_regs.cu: 8 warps x 10 KB per SM,
// 6.22 TB/s at 245,952 tokens x 40 heads); here a token's 20 KB waits in shared memory, so
// 8 resident CTAs of 256 threads (40 registers each) keep 160 KB in flight per SM, and as
// CTAs retire new ones start their copies while the others compute and store: 6.80 TB/s
// (128-thread CTAs: 6.73).
//
// Per CTA (T threads): thread 0 starts the two copies on one mbarrier; thread p < 64
// computes the token's position, pair p's (cos, sin) and its rotation coefficients with the
// q and k weights folded in (qk_coefs), into shared memory; then every thread takes vectors
// c = t + T u of the token's q | k vectors.  T is a multiple of the 16 vectors of a head vector, so thread t owns the same
// 8-element slice (8 * (t % 16) ..) of every head vector it touches and each head vector's
// sum of squares is one half-warp shuffle tree.  The per-slot arithmetic is qk_math.cuh's
// (bit-identical to k_qk_regs.cu's and k_qk_pool.cu's).  The wait on the copies is bounded;
// on give-up the CTA records bit 1 of the device error flags, waits once more (bounded) for
// its copies and returns.
#include <algorithm>
#include <atomic>

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "qk_math.cuh"

#ifndef SOL_QK_CTA_THREADS
#define SOL_QK_CTA_THREADS 256
#endif

namespace sol {

static __device__ unsigned int g_qk_error;

namespace {
constexpr int kQkCtaThreads = SOL_QK_CTA_THREADS;
constexpr uint32_t kQkWaitLimit = 4096;  // polls of <= ~1 ms each
}  // namespace

template <int U>
__global__ void __launch_bounds__(kQkCtaThreads)
    k_qk_cta(bf16* q_out, bf16* k_out, int64_t ld_qo, int64_t ld_ko, const bf16* q, const bf16* k, int64_t ld_q,
             int64_t ld_k, const bf16* __restrict__ wq, const bf16* __restrict__ wk, const int32_t* __restrict__ pos,
             int32_t grid_H, int32_t grid_W, uint32_t tokens_per_sample, RopeDev rope, int32_t n_heads, float eps)
{
    extern __shared__ __align__(128) uint4 rows[];  // [q row | k row], 2 * qv vectors
    __shared__ float4 kcs[2][4][16];  // rotation coefficients of pair 4 j + m at [q or k][m][j]
    __shared__ __align__(8) uint64_t bar;
    const uint32_t n = blockIdx.x;  // < 2^31 (checked on the host)
    const int t = threadIdx.x;
    const int qv = 16 * n_heads;    // 16-byte vectors of the q row (and of the k row)
    const uint32_t row_bytes = 16u * (uint32_t)qv;

    if (t == 0) {
        mbar_init(smem_u32(&bar), 1);
        mbar_fence_init();
        mbar_arrive_expect_tx(smem_u32(&bar), 2 * row_bytes);
        bulk_g2s(smem_u32(rows), q + (int64_t)n * ld_q, row_bytes, smem_u32(&bar));
        bulk_g2s(smem_u32(rows + qv), k + (int64_t)n * ld_k, row_bytes, smem_u32(&bar));
    }
    if (t < 64) {
        // the token's (t, h, w) position, then pair t's angle and its rotation coefficients
        // with the q and k weights folded in (qk_coefs of qk_math.cuh, per pair)
        uint32_t p0, p1, p2;
        if (pos) {
            p0 = (uint32_t)min(max(__ldg(pos + 3 * (int64_t)n + 0), 0), rope.max[0] - 1);
            p1 = (uint32_t)min(max(__ldg(pos + 3 * (int64_t)n + 1), 0), rope.max[1] - 1);
            p2 = (uint32_t)min(max(__ldg(pos + 3 * (int64_t)n + 2), 0), rope.max[2] - 1);
        } else {
            const uint32_t nl = tokens_per_sample ? n % tokens_per_sample : n;
            const uint32_t hw = (uint32_t)grid_H * (uint32_t)grid_W;
            p0 = nl / hw;
            const uint32_t r = nl - p0 * hw;
            p1 = r / (uint32_t)grid_W;
            p2 = r - p1 * (uint32_t)grid_W;
        }
        const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
        const float2* tp = t < h0    ? rope.tab[0] + (int64_t)p0 * rope.half[0] + t
                           : t < h01 ? rope.tab[1] + (int64_t)p1 * rope.half[1] + (t - h0)
                                     : rope.tab[2] + (int64_t)p2 * rope.half[2] + (t - h01);
        const float2 a = __ldg(tp);
#pragma unroll
        for (int isk = 0; isk < 2; ++isk) {
            const bf16* wrow = isk ? wk : wq;
            float w0 = 1.f, w1 = 1.f;
            if (wrow) {
                const __nv_bfloat162 wp = __ldg(reinterpret_cast<const __nv_bfloat162*>(wrow) + t);
                w0 = __low2float(wp);
                w1 = __high2float(wp);
            }
            kcs[isk][t & 3][t >> 2] = make_float4(w0 * a.x, w1 * a.y, w0 * a.y, w1 * a.x);
        }
    }
    __syncthreads();  // the barrier is initialised and the coefficients are in place

    // every thread waits (bounded) for the copies; the give-up decision is the CTA's
    const bool landed = mbar_wait_bounded(smem_u32(&bar), 0, kQkWaitLimit);
    if (__syncthreads_or(!landed)) {
        if (t == 0) {
            atomicOr(&g_qk_error, 2u);
            mbar_wait_bounded(smem_u32(&bar), 0, kQkWaitLimit);  // the copies must land before exit
        }
        return;
    }

    const int sub = t & 15;  // element slice 8 * sub .. + 7 of every head vector: pairs 4 sub ..
    // sums of squares and the half-warp trees of every slot (slots past the row are zero,
    // and uniform over each warp: T u + t and 2 * qv are multiples of 32)
    float ss[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        ss[u] = 0.f;
        const int c = t + kQkCtaThreads * u;
        if (c < 2 * qv) {
            float2 f[4];
            unpack2<bf16>(rows[c], f);
            ss[u] = qk_sumsq(f);
        }
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
        for (int u = 0; u < U; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c = t + kQkCtaThreads * u;
        if (c >= 2 * qv) continue;
        const bool isk = c >= qv;
        float kc[16];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 v = kcs[isk ? 1 : 0][m][sub];  // lanes read consecutive 16-byte words
            kc[4 * m + 0] = v.x;
            kc[4 * m + 1] = v.y;
            kc[4 * m + 2] = v.z;
            kc[4 * m + 3] = v.w;
        }
        float2 f[4];
        unpack2<bf16>(rows[c], f);
        float o[8];
        qk_rotate(f, rsqrtf(ss[u] * (1.f / 128.f) + eps), kc, o);
        bf16* dst = isk ? k_out + (int64_t)n * ld_ko + 8 * (c - qv) : q_out + (int64_t)n * ld_qo + 8 * c;
        st_stream(dst, pack<bf16>(o));
    }
}

namespace {

template <int U>
cudaError_t launch_u(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k, int64_t ld_q,
                     int64_t ld_k, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H, int32_t grid_W,
                     int64_t tps, const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    auto kern = k_qk_cta<U>;
    const size_t smem = (size_t)2 * 16 * 16 * n_heads;
    static std::atomic<size_t> attr_set[64];  // per device: the larger dynamic shared memory it allows
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (attr_set[dev].load(std::memory_order_acquire) < smem) {
        // the whole of the SM's unified L1 / shared memory as shared memory, so that the
        // thread limit (8 CTAs of 256), not the carveout, bounds the resident CTAs
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess && smem > 48 * 1024)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(smem, std::memory_order_release);
    }
    kern<<<(unsigned)n_tokens, kQkCtaThreads, smem, s>>>(
        static_cast<bf16*>(q_out), static_cast<bf16*>(k_out), ld_qo, ld_ko, static_cast<const bf16*>(q),
        static_cast<const bf16*>(k), ld_q, ld_k, static_cast<const bf16*>(wq), static_cast<const bf16*>(wk), pos,
        grid_H, grid_W, (uint32_t)tps, rope, n_heads, eps);
    return cudaGetLastError();
}

}  // namespace

bool qk_cta_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k, int64_t n_tokens)
{
    // the copies need 16-byte aligned rows (the API's rule) and at most 48 heads (U <= 12)
    return dt == SOL_DTYPE_BF16 && head_dim == 128 && n_heads >= 2 && n_heads % 2 == 0 && n_heads <= 48 && q && k &&
           n_tokens < ((int64_t)1 << 31);
}

cudaError_t launch_qk_cta(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                          int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                          int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                          int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_tokens == 0) return cudaSuccess;
    if (tps >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    switch ((32 * n_heads + kQkCtaThreads - 1) / kQkCtaThreads) {
#define SOL_QK_CTA_U(u)                                                                                           \
    case u:                                                                                                       \
        return launch_u<u>(q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, \
                           n_tokens, n_heads, eps, s);
        SOL_QK_CTA_U(1) SOL_QK_CTA_U(2) SOL_QK_CTA_U(3) SOL_QK_CTA_U(4) SOL_QK_CTA_U(5) SOL_QK_CTA_U(6)
        SOL_QK_CTA_U(7) SOL_QK_CTA_U(8) SOL_QK_CTA_U(9) SOL_QK_CTA_U(10) SOL_QK_CTA_U(11) SOL_QK_CTA_U(12)
#undef SOL_QK_CTA_U
    }
    return cudaErrorInvalidValue;
}

uint32_t qk_device_error(bool clear)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_qk_error, sizeof v) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_qk_error, &zero, sizeof zero);
    }
    return v;
}

}  // namespace sol
