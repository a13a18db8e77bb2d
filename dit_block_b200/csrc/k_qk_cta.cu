// k_qk_cta.cu -- QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合"]
// (bf16, head_dim 128, q and k both given) with one CTA per token whose q row and k row
// land in shared memory by two bulk asynchronous copies.
//
// Why: the op is an in-place stream of 4 bytes per element with little arithmetic, so it is
// bound by the bytes each SM keeps in flight.  Rows held in registers cap that at what the
// register file spares (a persistent warp per row, k_qk_regs.cu: 8 warps x 10 KB per SM,
// 6.22 TB/s at 245,952 tokens x 40 heads); here a token's 20 KB waits in shared memory, so
// 8 resident CTAs of 256 threads (32 registers each) keep 160 KB in flight per SM, and as
// CTAs retire new ones start their copies while the others compute and store: 6.80-6.91
// TB/s (128-thread CTAs: 6.73).
//
// Per CTA (T threads): thread 0 starts the two copies on one mbarrier; thread p < 64
// computes the token's position, pair p's (cos, sin) and its rotation coefficients with the
// q and k weights folded in (qk_coefs), into shared memory; then every thread takes vectors
// c = t + T u of the token's q | k vectors.  T is a multiple of the 16 vectors of a head
// vector, so thread t owns the same 8-element slice (8 * (t % 16) ..) of every head vector
// it touches and each head vector's sum of squares is one half-warp shuffle tree.  The
// per-slot arithmetic of the default convention is qk_math.cuh's (bit-identical to
// k_qk_regs.cu's and k_qk_pool.cu's).  The wait on the copies is bounded; on give-up the
// CTA records bit 1 of the device error flags, waits once more (bounded) for its copies and
// returns.
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

__device__ __forceinline__ void st_stream8(void* p, uint32_t x, uint32_t y)
{
    asm volatile("st.global.L1::no_allocate.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
}  // namespace

// Convention variants (sol_qk_rmsnorm_rope3d_ex) in the same kernel:
//   HALF     rotate-half pairs (element j of an axis chunk with element j + D_c / 2) in place
//            of interleaved ones, per head.  Pair p of a head vector has the angle of
//            interleaved pair p (index j within its axis chunk) and its two elements D_c / 2
//            apart; with chunk halves that are multiples of 4, thread `sub` takes pairs
//            4 sub .. 4 sub + 3: 4 consecutive first elements and their 4 partners, two
//            8-byte pieces of the staged row, written back as two 8-byte pieces.  The pair
//            coefficients (weights folded in) and the arithmetic are the interleaved ones.
//   ACROSS   one RMS over the whole q (k) row (interleaved pairs), weights [n_heads * 128]
//            laid out like the row: the slot sums meet in a CTA reduction (one barrier); the
//            weights differ per head, so they are read per slot (through L1), and the staged
//            table holds the bare (cos, sin).
//   STRIDED  outputs at (sample, token, head) element strides, e.g. [sample, head, token, dim].
// The default (per head, interleaved, token-major) is the plain op's path exactly.
template <int U, bool ACROSS, bool HALF, bool STRIDED>
__global__ void __launch_bounds__(kQkCtaThreads, 2048 / kQkCtaThreads)
    k_qk_cta(bf16* q_out, bf16* k_out, int64_t ld_qo, int64_t ld_ko, QkOutStrides os, const bf16* q, const bf16* k,
             int64_t ld_q, int64_t ld_k, const bf16* __restrict__ wq, const bf16* __restrict__ wk,
             const int32_t* __restrict__ pos, int32_t grid_H, int32_t grid_W, uint32_t tokens_per_sample, RopeDev rope,
             int32_t n_heads, float eps)
{
    static_assert(!(ACROSS && HALF), "rotate-half across heads runs on the row-in-registers kernel");
    extern __shared__ __align__(128) uint4 rows[];  // [q row | k row], 2 * qv vectors
    // per head: rotation coefficients of pair 4 j + m at [q or k][m][j], with the q, k
    // weights folded in; across heads: (cos, sin) of pair 4 j + m at [0][m][j].xy
    __shared__ float4 kcs[2][4][16];
    __shared__ float red[2][kQkCtaThreads / 32];
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
    const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
    if (t < 64) {
        // the token's (t, h, w) position, then pair t's angle: index j within its axis chunk
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
        const float2* tp = t < h0    ? rope.tab[0] + (int64_t)p0 * rope.half[0] + t
                           : t < h01 ? rope.tab[1] + (int64_t)p1 * rope.half[1] + (t - h0)
                                     : rope.tab[2] + (int64_t)p2 * rope.half[2] + (t - h01);
        const float2 a = __ldg(tp);
        if constexpr (ACROSS) {
            kcs[0][t & 3][t >> 2] = make_float4(a.x, a.y, 0.f, 0.f);
        } else {
            // the pair's two elements: (2 t, 2 t + 1), or rotate-half (e, e + D_c / 2)
            int ea = 2 * t, eb = 2 * t + 1;
            if constexpr (HALF) {
                const int hc = t < h0 ? rope.half[0] : (t < h01 ? rope.half[1] : rope.half[2]);
                ea = t < h0 ? t : (t < h01 ? t + h0 : t + h01);  // chunk start 2 (pairs before) + j
                eb = ea + hc;
            }
            // the q and k weights folded in (qk_coefs of qk_math.cuh, per pair)
#pragma unroll
            for (int isk = 0; isk < 2; ++isk) {
                const bf16* wrow = isk ? wk : wq;
                const float wa = wrow ? __bfloat162float(wrow[ea]) : 1.f;
                const float wb = wrow ? __bfloat162float(wrow[eb]) : 1.f;
                kcs[isk][t & 3][t >> 2] = make_float4(wa * a.x, wb * a.y, wa * a.y, wb * a.x);
            }
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

    const int sub = t & 15;  // pairs 4 sub .. 4 sub + 3 of every head vector the thread touches
    // sums of squares; per head: the half-warp trees of every slot (slots past the row are
    // zero, and uniform over each warp: T u + t and 2 * qv are multiples of 32); across
    // heads: one CTA reduction per row
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
    float r_row[2] = {0.f, 0.f};
    if constexpr (ACROSS) {
        float sq = 0.f, sk = 0.f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = t + kQkCtaThreads * u;
            if (c < qv)
                sq += ss[u];
            else
                sk += ss[u];
        }
        sq = warp_sum(sq);
        sk = warp_sum(sk);
        if ((t & 31) == 0) {
            red[0][t >> 5] = sq;
            red[1][t >> 5] = sk;
        }
        __syncthreads();
        float tq = 0.f, tk = 0.f;
#pragma unroll
        for (int w = 0; w < kQkCtaThreads / 32; ++w) {
            tq += red[0][w];
            tk += red[1][w];
        }
        const float inv = 1.f / (128.f * (float)n_heads);
        r_row[0] = rsqrtf(tq * inv + eps);
        r_row[1] = rsqrtf(tk * inv + eps);
    } else {
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
            for (int u = 0; u < U; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
        }
    }
    // rotate-half: this thread's first elements e0 .. e0 + 3 and their partners at + hp
    int e0 = 8 * sub, hp = 0;
    if constexpr (HALF) {
        const int p = 4 * sub;
        hp = p < h0 ? rope.half[0] : (p < h01 ? rope.half[1] : rope.half[2]);
        e0 = p < h0 ? p : (p < h01 ? p + h0 : p + h01);
    }
    // strided outputs: head 0 of the token, relative to q_out / k_out
    int64_t obase = 0;
    if constexpr (STRIDED) {
        const uint32_t sample = tokens_per_sample ? n / tokens_per_sample : 0;
        obase = (int64_t)sample * os.sample + (int64_t)(n - sample * tokens_per_sample) * os.token;
    }
    // (across heads no slot sum is needed any more: one slot at a time keeps registers low)
#pragma unroll(ACROSS ? 1 : U)
    for (int u = 0; u < U; ++u) {
        const int c = t + kQkCtaThreads * u;
        if (c >= 2 * qv) continue;
        const int isk = c >= qv ? 1 : 0;
        const int v = c - isk * qv;  // vector within the row: head v / 16, slice v % 16
        const int hh = v >> 4;
        float o[8];
        if constexpr (ACROSS) {
            // weights per slot, then the bare rotation
            const float r = isk ? r_row[1] : r_row[0];
            const bf16* wrow = isk ? wk : wq;
            float w[8];
            if (wrow) {
                unpack<bf16>(ld_cached(wrow + 8 * v), w);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) w[e] = 1.f;
            }
            float f[8], a[8];
            unpack<bf16>(rows[c], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) a[e] = f[e] * r * w[e];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 cssn = kcs[0][m][sub];
                o[2 * m] = a[2 * m] * cssn.x - a[2 * m + 1] * cssn.y;
                o[2 * m + 1] = a[2 * m] * cssn.y + a[2 * m + 1] * cssn.x;
            }
        } else {
            // the 4 pairs as (first, second) element, rotated with the folded coefficients
            float2 f[4];
            if constexpr (HALF) {
                const bf16* hrow = reinterpret_cast<const bf16*>(rows + (c - sub));  // the head vector
                const uint2 a = *reinterpret_cast<const uint2*>(hrow + e0);
                const uint2 b = *reinterpret_cast<const uint2*>(hrow + e0 + hp);
                f[0] = make_float2(bf_lo(a.x), bf_lo(b.x));
                f[1] = make_float2(bf_hi(a.x), bf_hi(b.x));
                f[2] = make_float2(bf_lo(a.y), bf_lo(b.y));
                f[3] = make_float2(bf_hi(a.y), bf_hi(b.y));
            } else {
                unpack2<bf16>(rows[c], f);
            }
            float kc[16];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 x = kcs[isk][m][sub];  // lanes read consecutive 16-byte words
                kc[4 * m + 0] = x.x;
                kc[4 * m + 1] = x.y;
                kc[4 * m + 2] = x.z;
                kc[4 * m + 3] = x.w;
            }
            qk_rotate(f, rsqrtf(ss[u] * (1.f / 128.f) + eps), kc, o);
        }
        bf16* dst;  // the head vector's output
        if constexpr (STRIDED) {
            dst = (isk ? k_out : q_out) + obase + (int64_t)hh * os.head;
        } else {
            dst = isk ? k_out + (int64_t)n * ld_ko + 128 * hh : q_out + (int64_t)n * ld_qo + 128 * hh;
        }
        if constexpr (HALF) {
            st_stream8(dst + e0, pack2_bf16(o[0], o[2]), pack2_bf16(o[4], o[6]));
            st_stream8(dst + e0 + hp, pack2_bf16(o[1], o[3]), pack2_bf16(o[5], o[7]));
        } else {
            st_stream(dst + 8 * sub, pack<bf16>(o));
        }
    }
    (void)r_row;
    (void)hp;
}

namespace {

template <int U, bool ACROSS, bool HALF, bool STRIDED>
cudaError_t launch_u(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const QkOutStrides& os, const void* q,
                     const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                     int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                     int32_t n_heads, float eps, cudaStream_t s)
{
    auto kern = k_qk_cta<U, ACROSS, HALF, STRIDED>;
    const size_t smem = (size_t)2 * 16 * 16 * n_heads;
    static std::atomic<size_t> attr_set[64];  // per device: the larger dynamic shared memory it allows
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (attr_set[dev].load(std::memory_order_acquire) < smem) {
        // enough of the SM's unified L1 / shared memory as shared memory that the thread
        // limit (8 CTAs of 256), not the carveout, bounds the resident CTAs: all of it, or
        // for the across-heads variants, which read their weights per slot through L1, just
        // enough (per CTA: the row, ~2 KB of static arrays and the 1 KB the system keeps)
        int carveout = (int)cudaSharedmemCarveoutMaxShared;
        if (ACROSS) {
            const size_t need = (smem + 3 * 1024) * (2048 / kQkCtaThreads);
            carveout = (int)std::min<size_t>(100, (need * 100 + 228 * 1024 - 1) / (228 * 1024));
        }
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, carveout);
        if (e == cudaSuccess && smem > 48 * 1024)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(smem, std::memory_order_release);
    }
    kern<<<(unsigned)n_tokens, kQkCtaThreads, smem, s>>>(
        static_cast<bf16*>(q_out), static_cast<bf16*>(k_out), ld_qo, ld_ko, os, static_cast<const bf16*>(q),
        static_cast<const bf16*>(k), ld_q, ld_k, static_cast<const bf16*>(wq), static_cast<const bf16*>(wk), pos,
        grid_H, grid_W, (uint32_t)tps, rope, n_heads, eps);
    return cudaGetLastError();
}

template <bool ACROSS, bool HALF, bool STRIDED>
cudaError_t dispatch_u(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const QkOutStrides& os, const void* q,
                       const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                       int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                       int32_t n_heads, float eps, cudaStream_t s)
{
    switch ((32 * n_heads + kQkCtaThreads - 1) / kQkCtaThreads) {
#define SOL_QK_CTA_U(u)                                                                                        \
    case u:                                                                                                    \
        return launch_u<u, ACROSS, HALF, STRIDED>(q_out, k_out, ld_qo, ld_ko, os, q, k, ld_q, ld_k, wq, wk, pos, \
                                                  grid_H, grid_W, tps, rope, n_tokens, n_heads, eps, s);
        SOL_QK_CTA_U(1) SOL_QK_CTA_U(2) SOL_QK_CTA_U(3) SOL_QK_CTA_U(4) SOL_QK_CTA_U(5) SOL_QK_CTA_U(6)
#undef SOL_QK_CTA_U
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool qk_cta_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k, int64_t n_tokens)
{
    // the copies need 16-byte aligned rows (the API's rule); 256 threads cover up to 48 heads
    // with 6 vectors each
    return dt == SOL_DTYPE_BF16 && head_dim == 128 && n_heads >= 2 && n_heads % 2 == 0 && n_heads <= 48 && q && k &&
           n_tokens < ((int64_t)1 << 31);
}

namespace {
// token-major outputs (head stride 128, samples back to back) take the unstrided stores
bool out_token_major(const QkOutStrides& os, int64_t tps, int64_t n_tokens)
{
    const int64_t tps_eff = tps > 0 ? tps : n_tokens;
    return os.head == 128 && (os.sample == tps_eff * os.token || n_tokens <= tps_eff);
}
}  // namespace

bool qk_cta_ex_fits(sol_dtype dt, bool across, bool half, int32_t n_heads, int32_t head_dim,
                    const void* q, const void* k, int64_t n_tokens, int64_t tps, const RopeDev& rope)
{
    if (!qk_cta_fits(dt, n_heads, head_dim, q, k, n_tokens) || tps >= ((int64_t)1 << 31)) return false;
    if (half) {
        // rotate-half per head only: across heads the row-in-registers kernel measured faster
        // (and one kernel serves every output layout, so results do not depend on the layout)
        if (across) return false;
        for (int c = 0; c < 3; ++c)
            if (rope.half[c] % 4 != 0) return false;
    }
    return true;
}

cudaError_t launch_qk_cta(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                          int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                          int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                          int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_tokens == 0) return cudaSuccess;
    if (tps >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const QkOutStrides os{0, 0, 0};  // unused: token-major outputs
    return dispatch_u<false, false, false>(q_out, k_out, ld_qo, ld_ko, os, q, k, ld_q, ld_k, wq, wk, pos, grid_H,
                                           grid_W, tps, rope, n_tokens, n_heads, eps, s);
}

cudaError_t launch_qk_cta_ex(bool across, bool half, void* q_out, void* k_out, const QkOutStrides& os, const void* q,
                             const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk,
                             const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope,
                             int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_tokens == 0) return cudaSuccess;
    if (half && across) return cudaErrorInvalidValue;  // outside qk_cta_ex_fits
    const bool token_major = out_token_major(os, tps, n_tokens);
    const int64_t ld_o = os.token;
#define SOL_QK_CTA_EX_ARGS q_out, k_out, ld_o, ld_o, os, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, n_tokens, n_heads, eps, s
    if (token_major) {
        if (half) return dispatch_u<false, true, false>(SOL_QK_CTA_EX_ARGS);
        return across ? dispatch_u<true, false, false>(SOL_QK_CTA_EX_ARGS)
                      : dispatch_u<false, false, false>(SOL_QK_CTA_EX_ARGS);
    }
    if (half) return dispatch_u<false, true, true>(SOL_QK_CTA_EX_ARGS);
    return across ? dispatch_u<true, false, true>(SOL_QK_CTA_EX_ARGS)
                  : dispatch_u<false, false, true>(SOL_QK_CTA_EX_ARGS);
#undef SOL_QK_CTA_EX_ARGS
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
