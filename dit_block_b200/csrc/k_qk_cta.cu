// k_qk_cta.cu -- QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合"]
// (bf16, head_dim 128, q and k both given) with one CTA per token whose q row and k row
// land in shared memory by two bulk asynchronous copies.
//
// Why: the op is an in-place stream of 4 bytes per element with little arithmetic, so it is
// bound by the bytes each SM keeps in flight.  Rows held in registers cap that at what the
// register file spares (a persistent warp per row, k_qk_regs.cu: 8 warps x 10 KB per SM,
// 6.22 TB/s at 245,952 tokens x 40 heads); here a token's 20 KB waits in shared memory, and
// as CTAs retire new ones start their copies while the others compute and store.
//
// k_qk_head (the plain op and every convention of sol_qk_rmsnorm_rope3d_ex): 128 threads, 9
// resident CTAs per SM (shared memory bounds them: 9 x 22.6 KB = 180 KB in flight), 48-56
// registers.  The q row is done, then the k row; a thread takes vectors t + 128 u of the row
// and keeps the row's 16 rotation coefficients of its slice in registers for all of them.
// 6.8-6.9 TB/s alone and inside the block pass, also at
// the 1.5 GHz the power cap holds in long runs (an earlier 256-thread form that read its
// coefficients from shared memory per vector streamed 6.9 alone but 6.0 there: its
// shared-memory pipe ran near full, and its compute phase, which holds the CTA's rows,
// followed the clock).
//
// Per CTA: thread 0 starts the two copies on one mbarrier; thread p < 64 computes the
// token's position, pair p's (cos, sin) and, per head, its rotation coefficients with the q
// and k weights folded in (qk_coefs), into shared memory.  128 is a multiple of the 16
// vectors of a head vector, so thread t owns the same 8-element slice
// (8 * (t % 16) ..) of every head vector it touches and each head vector's sum of squares
// is one half-warp shuffle tree.  The per-slot arithmetic of the default convention is
// qk_math.cuh's (bit-identical to k_qk_regs.cu's and k_qk_pool.cu's).  The wait on the
// copies is bounded; on give-up the CTA records bit 1 of the device error flags, waits once
// more (bounded) for its copies and returns.
#include <algorithm>
#include <atomic>

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "qk_math.cuh"

namespace sol {

static __device__ unsigned int g_qk_error;

namespace {
constexpr int kHeadThreads = 128;        // k_qk_head
constexpr int kHeadCtas = 9;             // resident k_qk_head CTAs per SM (launch bounds)
constexpr uint32_t kQkWaitLimit = 4096;  // polls of <= ~1 ms each

__device__ __forceinline__ void st_stream8(void* p, uint32_t x, uint32_t y)
{
    asm volatile("st.global.L1::no_allocate.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(x), "r"(y) : "memory");
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Thread 0: start the bulk copies of the token's q and k rows (16 * qv bytes each).
__device__ __forceinline__ void start_row_copies(uint4* rows, uint64_t* bar, const bf16* q, const bf16* k,
                                                 int64_t ld_q, int64_t ld_k, uint32_t n, int qv)
{
    const uint32_t row_bytes = 16u * (uint32_t)qv;
    mbar_init(smem_u32(bar), 1);
    mbar_fence_init();
    mbar_arrive_expect_tx(smem_u32(bar), 2 * row_bytes);
    bulk_g2s(smem_u32(rows), q + (int64_t)n * ld_q, row_bytes, smem_u32(bar));
    bulk_g2s(smem_u32(rows + qv), k + (int64_t)n * ld_k, row_bytes, smem_u32(bar));
}

// Pair p's (cos, sin) for token n: its axis chunk, the token's position on that axis (from
// pos, clamped to the table, or from the token's place in its sample's T x H x W grid) and
// the pair's index j within the chunk.
__device__ __forceinline__ float2 pair_angle(int p, uint32_t n, const int32_t* __restrict__ pos, int32_t grid_H,
                                             int32_t grid_W, uint32_t tokens_per_sample, RopeDev rope)
{
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
    const float2* tp = p < h0    ? rope.tab[0] + (int64_t)p0 * rope.half[0] + p
                       : p < h01 ? rope.tab[1] + (int64_t)p1 * rope.half[1] + (p - h0)
                                 : rope.tab[2] + (int64_t)p2 * rope.half[2] + (p - h01);
    return __ldg(tp);
}

// Every thread waits (bounded) for the copies; the give-up decision is the CTA's.  Returns
// false (after recording the error and draining the copies) when the CTA must exit.
__device__ __forceinline__ bool rows_landed(uint64_t* bar)
{
    const bool landed = mbar_wait_bounded(smem_u32(bar), 0, kQkWaitLimit);
    if (__syncthreads_or(!landed)) {
        if (threadIdx.x == 0) {
            atomicOr(&g_qk_error, 2u);
            mbar_wait_bounded(smem_u32(bar), 0, kQkWaitLimit);  // the copies must land before exit
        }
        return false;
    }
    return true;
}
}  // namespace

// UQ = vectors per thread and row.  The default (per head, interleaved pairs, token-major
// rows) is the plain op.
//   ACROSS   one RMS over the whole q (k) row, weights [n_heads * 128] laid out like the
//            row: the thread sums of the two rows meet in one CTA reduction (one barrier);
//            the weights differ per head, so each vector's are read (through L1) and
//            multiply its elements before a rotation with the bare (cos, sin).
//   HALF     rotate-half pairs (element j of an axis chunk with element j + D_c / 2) in
//            place of interleaved ones.  Pair p of a head vector has the angle of interleaved
//            pair p (index j within its axis chunk) and its two elements D_c / 2 apart, so
//            the pair coefficients and the arithmetic are the interleaved ones; with chunk
//            halves that are multiples of 4, thread `sub` takes pairs 4 sub .. 4 sub + 3: 4
//            consecutive first elements and their 4 partners, two 8-byte pieces of the
//            staged row, written back as two 8-byte pieces.
//   STRIDED  outputs at (sample, token, head) element strides, e.g. [sample, head, token, dim].
template <int UQ, bool ACROSS, bool HALF, bool STRIDED>
__global__ void __launch_bounds__(kHeadThreads, kHeadCtas)
    k_qk_head(bf16* q_out, bf16* k_out, int64_t ld_qo, int64_t ld_ko, QkOutStrides os, const bf16* q, const bf16* k,
              int64_t ld_q, int64_t ld_k, const bf16* __restrict__ wq, const bf16* __restrict__ wk,
              const int32_t* __restrict__ pos, int32_t grid_H, int32_t grid_W, uint32_t tokens_per_sample,
              RopeDev rope, int32_t n_heads, float eps)
{
    extern __shared__ __align__(128) uint4 rows[];  // [q row | k row], 2 * qv vectors
    // rotation coefficients of pair 4 j + m at [q or k][m][j], weights folded in; across
    // heads [0][m][j], without weights
    __shared__ float4 kcs[2][4][16];
    __shared__ float red[2][kHeadThreads / 32];
    __shared__ __align__(8) uint64_t bar;
    const uint32_t n = blockIdx.x;  // < 2^31 (checked on the host)
    const int t = threadIdx.x;
    const int qv = 16 * n_heads;    // 16-byte vectors of the q row (and of the k row)

    if (t == 0) start_row_copies(rows, &bar, q, k, ld_q, ld_k, n, qv);
    const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
    if (ACROSS && t < 64) {
        const float2 a = pair_angle(t, n, pos, grid_H, grid_W, tokens_per_sample, rope);
        kcs[0][t & 3][t >> 2] = make_float4(a.x, a.y, a.y, a.x);
    } else if (t < 64) {
        const float2 a = pair_angle(t, n, pos, grid_H, grid_W, tokens_per_sample, rope);
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
    __syncthreads();  // the barrier is initialised and the coefficients are in place
    if (!rows_landed(&bar)) return;

    const int sub = t & 15;  // pairs 4 sub .. 4 sub + 3 of every head vector the thread touches
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
    float r_row[2] = {0.f, 0.f};
    if constexpr (ACROSS) {
        float sr[2] = {0.f, 0.f};
#pragma unroll
        for (int isk = 0; isk < 2; ++isk) {
#pragma unroll
            for (int u = 0; u < UQ; ++u) {
                const int c = t + kHeadThreads * u;
                if (c < qv) {
                    float2 f[4];
                    unpack2<bf16>(rows[isk * qv + c], f);
                    sr[isk] += qk_sumsq(f);
                }
            }
            sr[isk] = warp_sum(sr[isk]);
        }
        if ((t & 31) == 0) {
            red[0][t >> 5] = sr[0];
            red[1][t >> 5] = sr[1];
        }
        __syncthreads();
        const float inv = 1.f / (128.f * (float)n_heads);
#pragma unroll
        for (int isk = 0; isk < 2; ++isk) {
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < kHeadThreads / 32; ++w) tot += red[isk][w];
            r_row[isk] = rsqrtf(tot * inv + eps);
        }
    }
#pragma unroll
    for (int isk = 0; isk < 2; ++isk) {
        const uint4* row = rows + isk * qv;
        // sums of squares of the head vectors: the half-warp tree of every slot (slots past
        // the row are zero, and uniform over each warp: qv is a multiple of 32)
        float ss[UQ];
#pragma unroll
        for (int u = 0; u < UQ; ++u) {
            ss[u] = 0.f;
            const int c = t + kHeadThreads * u;
            if (!ACROSS && c < qv) {
                float2 f[4];
                unpack2<bf16>(row[c], f);
                ss[u] = qk_sumsq(f);
            }
        }
        if constexpr (!ACROSS) {
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
                for (int u = 0; u < UQ; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
            }
        }
        float kc[16];  // this slice's coefficients, for every head vector of the row
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 x = kcs[ACROSS ? 0 : isk][m][sub];  // lanes read consecutive 16-byte words
            kc[4 * m + 0] = x.x;
            kc[4 * m + 1] = x.y;
            kc[4 * m + 2] = x.z;
            kc[4 * m + 3] = x.w;
        }
        bf16* const out = isk ? k_out : q_out;
#pragma unroll
        for (int u = 0; u < UQ; ++u) {
            const int c = t + kHeadThreads * u;
            if (c >= qv) continue;
            // the 4 pairs as (first, second) element
            float2 f[4];
            if constexpr (HALF) {
                const bf16* hrow = reinterpret_cast<const bf16*>(row + (c - sub));  // the head vector
                const uint2 a = *reinterpret_cast<const uint2*>(hrow + e0);
                const uint2 b = *reinterpret_cast<const uint2*>(hrow + e0 + hp);
                f[0] = make_float2(bf_lo(a.x), bf_lo(b.x));
                f[1] = make_float2(bf_hi(a.x), bf_hi(b.x));
                f[2] = make_float2(bf_lo(a.y), bf_lo(b.y));
                f[3] = make_float2(bf_hi(a.y), bf_hi(b.y));
            } else {
                unpack2<bf16>(row[c], f);
            }
            if constexpr (ACROSS) {
                // the weights of these elements (per head, so per slot), before the rotation
                const bf16* wrow = isk ? wk : wq;
                if (wrow) {
                    float2 w[4];
                    if constexpr (HALF) {
                        const bf16* wh = wrow + 8 * (c - sub);
                        const uint2 a = __ldg(reinterpret_cast<const uint2*>(wh + e0));
                        const uint2 b = __ldg(reinterpret_cast<const uint2*>(wh + e0 + hp));
                        w[0] = make_float2(bf_lo(a.x), bf_lo(b.x));
                        w[1] = make_float2(bf_hi(a.x), bf_hi(b.x));
                        w[2] = make_float2(bf_lo(a.y), bf_lo(b.y));
                        w[3] = make_float2(bf_hi(a.y), bf_hi(b.y));
                    } else {
                        unpack2<bf16>(ld_cached(wrow + 8 * c), w);
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) f[m] = __fmul2_rn(f[m], w[m]);
                }
            }
            float o[8];
            qk_rotate(f, ACROSS ? r_row[isk] : rsqrtf(ss[u] * (1.f / 128.f) + eps), kc, o);
            bf16* dst;  // the head vector's output
            if constexpr (STRIDED)
                dst = out + obase + (int64_t)(c >> 4) * os.head;
            else
                dst = out + (int64_t)n * (isk ? ld_ko : ld_qo) + 8 * (c - sub);
            if constexpr (HALF) {
                st_stream8(dst + e0, pack2_bf16(o[0], o[2]), pack2_bf16(o[4], o[6]));
                st_stream8(dst + e0 + hp, pack2_bf16(o[1], o[3]), pack2_bf16(o[5], o[7]));
            } else {
                st_stream(dst + 8 * sub, pack<bf16>(o));
            }
        }
    }
    (void)hp;
    (void)r_row;
}

namespace {

// Launch arguments.
struct QkLaunch {
    void* q_out;
    void* k_out;
    int64_t ld_qo, ld_ko;
    QkOutStrides os;
    const void* q;
    const void* k;
    int64_t ld_q, ld_k;
    const void* wq;
    const void* wk;
    const int32_t* pos;
    int32_t grid_H, grid_W;
    int64_t tps;
    RopeDev rope;
    int64_t n_tokens;
    int32_t n_heads;
    float eps;
};

// Set the kernel's shared-memory attributes once per device (for the largest row seen:
// all of the unified L1 / shared memory as shared memory, since 9 CTAs of 22.6 KB need it),
// then launch one CTA per token.
template <typename Kern>
cudaError_t launch_rows(Kern kern, const QkLaunch& a, std::atomic<size_t>* attr_set, cudaStream_t s)
{
    const size_t smem = (size_t)2 * 16 * 16 * a.n_heads;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (attr_set[dev].load(std::memory_order_acquire) < smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess && smem > 48 * 1024)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(smem, std::memory_order_release);
    }
    kern<<<(unsigned)a.n_tokens, kHeadThreads, smem, s>>>(
        static_cast<bf16*>(a.q_out), static_cast<bf16*>(a.k_out), a.ld_qo, a.ld_ko, a.os,
        static_cast<const bf16*>(a.q), static_cast<const bf16*>(a.k), a.ld_q, a.ld_k, static_cast<const bf16*>(a.wq),
        static_cast<const bf16*>(a.wk), a.pos, a.grid_H, a.grid_W, (uint32_t)a.tps, a.rope, a.n_heads, a.eps);
    return cudaGetLastError();
}

template <int UQ, bool ACROSS, bool HALF, bool STRIDED> cudaError_t launch_head(const QkLaunch& a, cudaStream_t s)
{
    static std::atomic<size_t> attr_set[64];  // per device: the larger dynamic shared memory it allows
    return launch_rows(k_qk_head<UQ, ACROSS, HALF, STRIDED>, a, attr_set, s);
}

template <bool ACROSS, bool HALF, bool STRIDED> cudaError_t dispatch_head(const QkLaunch& a, cudaStream_t s)
{
    switch ((16 * a.n_heads + kHeadThreads - 1) / kHeadThreads) {
    case 1: return launch_head<1, ACROSS, HALF, STRIDED>(a, s);
    case 2: return launch_head<2, ACROSS, HALF, STRIDED>(a, s);
    case 3: return launch_head<3, ACROSS, HALF, STRIDED>(a, s);
    case 4: return launch_head<4, ACROSS, HALF, STRIDED>(a, s);
    case 5: return launch_head<5, ACROSS, HALF, STRIDED>(a, s);
    case 6: return launch_head<6, ACROSS, HALF, STRIDED>(a, s);
    }
    return cudaErrorInvalidValue;
}

// token-major outputs (head stride 128, samples back to back) take the unstrided stores
bool out_token_major(const QkOutStrides& os, int64_t tps, int64_t n_tokens)
{
    const int64_t tps_eff = tps > 0 ? tps : n_tokens;
    return os.head == 128 && (os.sample == tps_eff * os.token || n_tokens <= tps_eff);
}

}  // namespace

bool qk_cta_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k, int64_t n_tokens)
{
    // the copies need 16-byte aligned rows (the API's rule); 128 threads cover up to 48 heads
    // with 6 vectors a thread and row
    return dt == SOL_DTYPE_BF16 && head_dim == 128 && n_heads >= 2 && n_heads % 2 == 0 && n_heads <= 48 && q && k &&
           n_tokens < ((int64_t)1 << 31);
}

bool qk_cta_ex_fits(sol_dtype dt, bool half, int32_t n_heads, int32_t head_dim,
                    const void* q, const void* k, int64_t n_tokens, int64_t tps, const RopeDev& rope)
{
    if (!qk_cta_fits(dt, n_heads, head_dim, q, k, n_tokens) || tps >= ((int64_t)1 << 31)) return false;
    if (half)  // a thread's 4 pairs in one chunk half, its pieces 8-byte aligned
        for (int c = 0; c < 3; ++c)
            if (rope.half[c] % 4 != 0) return false;
    return true;
}

cudaError_t launch_qk_cta(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                          int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                          int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                          int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_tokens == 0) return cudaSuccess;
    if (tps >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const QkLaunch a{q_out, k_out, ld_qo, ld_ko, QkOutStrides{0, 0, 0}, q, k, ld_q, ld_k, wq, wk, pos,
                     grid_H, grid_W, tps, rope, n_tokens, n_heads, eps};
    return dispatch_head<false, false, false>(a, s);
}

cudaError_t launch_qk_cta_ex(bool across, bool half, void* q_out, void* k_out, const QkOutStrides& os, const void* q,
                             const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk,
                             const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope,
                             int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_tokens == 0) return cudaSuccess;
    if (tps >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
    const bool token_major = out_token_major(os, tps, n_tokens);
    const QkLaunch a{q_out, k_out, os.token, os.token, os, q, k, ld_q, ld_k, wq, wk, pos,
                     grid_H, grid_W, tps, rope, n_tokens, n_heads, eps};
    if (across && half) return token_major ? dispatch_head<true, true, false>(a, s) : dispatch_head<true, true, true>(a, s);
    if (across) return token_major ? dispatch_head<true, false, false>(a, s) : dispatch_head<true, false, true>(a, s);
    if (half) return token_major ? dispatch_head<false, true, false>(a, s) : dispatch_head<false, true, true>(a, s);
    return token_major ? dispatch_head<false, false, false>(a, s) : dispatch_head<false, false, true>(a, s);
}

// ---------------------------------------------------------------------------------
// The QKV epilogue fused with the 64-token block means of SubBlock routing
// (sol_dit_epilogue_pool), staged: one CTA of 128 threads per (block, q or k) walks the
// block's tokens through a ring of kPoolSlots row buffers that thread 0 refills by bulk
// copies as rows are consumed, so up to kPoolSlots rows per CTA (4 CTAs per SM) are in
// flight while the block sums stay in fp32 registers.  Thread t owns vectors t + 128 u of
// the row (the same 8-element slice of every head vector it touches) and the 4 rotary
// pairs of that slice: its coefficients are recomputed per token from its weights and the
// token's angles (qk_coefs), and the per-vector arithmetic is qk_math.cuh's, so the
// in-place rows equal the plain epilogue's bit for bit and the sums are taken over the
// same fp32 outputs, token by token.  Every wait on a row is bounded; on give-up the CTA
// records bit 1 of the device error flags, waits (bounded) for its copies in flight and
// returns.
constexpr int kPoolSlots = 4;
constexpr int kPoolCtas = 4;  // resident CTAs per SM (launch bounds)

template <int UQ>
__global__ void __launch_bounds__(kHeadThreads, kPoolCtas)
    k_qk_pool_stage(bf16* q, bf16* k, int64_t ld_q, int64_t ld_k, bf16* pq, bf16* pk, int64_t ld_pq, int64_t ld_pk,
                    const bf16* __restrict__ wq, const bf16* __restrict__ wk, const int32_t* __restrict__ pos,
                    int32_t grid_H, int32_t grid_W, int64_t tps, int32_t block, int64_t bps, RopeDev rope,
                    int64_t n_tokens, int32_t n_heads, float eps)
{
    extern __shared__ __align__(128) uint4 ring[];  // kPoolSlots rows of qv vectors
    __shared__ __align__(8) uint64_t full[kPoolSlots];
    const int t = threadIdx.x;
    const int sub = t & 15;
    const int qv = 16 * n_heads;
    const uint32_t row_bytes = 16u * (uint32_t)qv;
    const int64_t blk = (int64_t)(blockIdx.x >> 1);
    const bool isk = (blockIdx.x & 1) != 0;
    // the block's tokens [t0, t1): blocks restart at every sample boundary
    const int64_t sample = blk / bps;
    const int64_t t0 = sample * tps + (blk - sample * bps) * block;
    int64_t t1 = t0 + block;
    if (t1 > (sample + 1) * tps) t1 = (sample + 1) * tps;
    if (t1 > n_tokens) t1 = n_tokens;
    const int cnt = (int)(t1 - t0);
    if (cnt <= 0) return;  // no block is empty (the host counts them); uniform over the CTA
    bf16* const rows_g = isk ? k : q;
    const int64_t ld = isk ? ld_k : ld_q;

    if (t == 0) {
#pragma unroll
        for (int i = 0; i < kPoolSlots; ++i) mbar_init(smem_u32(&full[i]), 1);
        mbar_fence_init();
        for (int i = 0; i < kPoolSlots && i < cnt; ++i) {
            mbar_arrive_expect_tx(smem_u32(&full[i]), row_bytes);
            bulk_g2s(smem_u32(ring + i * qv), rows_g + (t0 + i) * ld, row_bytes, smem_u32(&full[i]));
        }
    }
    // this slice's weights, and its 4 pairs' axis, table column and table row stride
    float w[8];
    const bf16* wsrc = isk ? wk : wq;
    if (wsrc) {
        unpack<bf16>(ld_cached(wsrc + 8 * sub), w);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = 1.f;
    }
    const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
    int axis[4];
    const float2* tb[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int pi = 4 * sub + m;
        axis[m] = pi < h0 ? 0 : (pi < h01 ? 1 : 2);
        tb[m] = axis[m] == 0 ? rope.tab[0] + pi : (axis[m] == 1 ? rope.tab[1] + (pi - h0) : rope.tab[2] + (pi - h01));
    }
    // the grid position of the next token (implicit positions)
    uint32_t g0 = 0, g1 = 0, g2 = 0;
    if (!pos) {
        const uint32_t nl = (uint32_t)(t0 - sample * tps);
        const uint32_t hw = (uint32_t)grid_H * (uint32_t)grid_W;
        g0 = nl / hw;
        const uint32_t r = nl - g0 * hw;
        g1 = r / (uint32_t)grid_W;
        g2 = r - g1 * (uint32_t)grid_W;
    }
    float acc[UQ][8];
#pragma unroll
    for (int u = 0; u < UQ; ++u)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
    __syncthreads();  // the barriers are initialised

    for (int i = 0; i < cnt; ++i) {
        const int slot = i % kPoolSlots;
        const bool landed = mbar_wait_bounded(smem_u32(&full[slot]), (uint32_t)(i / kPoolSlots) & 1u, kQkWaitLimit);
        if (__syncthreads_or(!landed)) {
            if (t == 0) {
                atomicOr(&g_qk_error, 2u);
                for (int j = i; j < cnt && j < i + kPoolSlots; ++j)  // the copies in flight must land
                    mbar_wait_bounded(smem_u32(&full[j % kPoolSlots]), (uint32_t)(j / kPoolSlots) & 1u,
                                      kQkWaitLimit);
            }
            return;
        }
        const int64_t n = t0 + i;
        uint32_t p[3];
        if (pos) {
            p[0] = (uint32_t)min(max(__ldg(pos + 3 * n + 0), 0), rope.max[0] - 1);
            p[1] = (uint32_t)min(max(__ldg(pos + 3 * n + 1), 0), rope.max[1] - 1);
            p[2] = (uint32_t)min(max(__ldg(pos + 3 * n + 2), 0), rope.max[2] - 1);
        } else {
            p[0] = g0;
            p[1] = g1;
            p[2] = g2;
            if (++g2 == (uint32_t)grid_W) {
                g2 = 0;
                if (++g1 == (uint32_t)grid_H) {
                    g1 = 0;
                    ++g0;
                }
            }
        }
        float cs[4], sn[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const uint32_t pm = axis[m] == 0 ? p[0] : (axis[m] == 1 ? p[1] : p[2]);
            const int st = axis[m] == 0 ? rope.half[0] : (axis[m] == 1 ? rope.half[1] : rope.half[2]);
            const float2 a = __ldg(tb[m] + (int64_t)pm * st);
            cs[m] = a.x;
            sn[m] = a.y;
        }
        float kc[16];
        qk_coefs(w, cs, sn, kc);
        const uint4* row = ring + slot * qv;
        float ss[UQ];
#pragma unroll
        for (int u = 0; u < UQ; ++u) {
            ss[u] = 0.f;
            const int c = t + kHeadThreads * u;
            if (c < qv) {
                float2 f[4];
                unpack2<bf16>(row[c], f);
                ss[u] = qk_sumsq(f);
            }
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
            for (int u = 0; u < UQ; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
        }
        bf16* const dst = rows_g + n * ld;
#pragma unroll
        for (int u = 0; u < UQ; ++u) {
            const int c = t + kHeadThreads * u;
            if (c >= qv) continue;
            float2 f[4];
            unpack2<bf16>(row[c], f);
            float o[8];
            qk_rotate(f, rsqrtf(ss[u] * (1.f / 128.f) + eps), kc, o);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[u][e] += o[e];
            st_stream(dst + 8 * c, pack<bf16>(o));
        }
        __syncthreads();  // every thread is done with the slot
        if (t == 0 && i + kPoolSlots < cnt) {
            mbar_arrive_expect_tx(smem_u32(&full[slot]), row_bytes);
            bulk_g2s(smem_u32(ring + slot * qv), rows_g + (n + kPoolSlots) * ld, row_bytes, smem_u32(&full[slot]));
        }
    }
    const float inv = 1.f / (float)cnt;
    bf16* const out = isk ? pk + blk * ld_pk : pq + blk * ld_pq;
#pragma unroll
    for (int u = 0; u < UQ; ++u) {
        const int c = t + kHeadThreads * u;
        if (c >= qv) continue;
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = acc[u][e] * inv;
        st_stream(out + 8 * c, pack<bf16>(o));
    }
}

namespace {
template <int UQ>
cudaError_t launch_pool_stage(void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk, int64_t ld_pq,
                              int64_t ld_pk, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                              int32_t grid_W, int64_t tps, int32_t block, int64_t bps, int64_t n_blocks,
                              const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    auto kern = k_qk_pool_stage<UQ>;
    const size_t smem = (size_t)kPoolSlots * 16 * 16 * n_heads;  // up to 48 KB (48 heads)
    static std::atomic<size_t> attr_set[64];  // per device: the larger dynamic shared memory it allows
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (attr_set[dev].load(std::memory_order_acquire) < smem) {
        // 4 CTAs of up to 48 KB: all of the unified L1 / shared memory as shared memory; the
        // dynamic part plus the barriers may pass the 48 KB a launch gets without asking
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev].store(smem, std::memory_order_release);
    }
    kern<<<(unsigned)(2 * n_blocks), kHeadThreads, smem, s>>>(
        static_cast<bf16*>(q), static_cast<bf16*>(k), ld_q, ld_k, static_cast<bf16*>(pq), static_cast<bf16*>(pk),
        ld_pq, ld_pk, static_cast<const bf16*>(wq), static_cast<const bf16*>(wk), pos, grid_H, grid_W, tps, block,
        bps, rope, n_tokens, n_heads, eps);
    return cudaGetLastError();
}
}  // namespace

bool qk_pool_stage_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k,
                        int64_t tps, int64_t n_blocks)
{
    return dt == SOL_DTYPE_BF16 && head_dim == 128 && n_heads >= 2 && n_heads % 2 == 0 && n_heads <= 48 && q && k &&
           tps < ((int64_t)1 << 31) && 2 * n_blocks < ((int64_t)1 << 31);
}

cudaError_t launch_qk_pool_stage(void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk, int64_t ld_pq,
                                 int64_t ld_pk, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                                 int32_t grid_W, int64_t tps, int32_t block, int64_t bps, int64_t n_blocks,
                                 const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    if (n_blocks == 0) return cudaSuccess;
    switch ((16 * n_heads + kHeadThreads - 1) / kHeadThreads) {
#define SOL_POOL_STAGE_U(u)                                                                                      \
    case u:                                                                                                      \
        return launch_pool_stage<u>(q, k, ld_q, ld_k, pq, pk, ld_pq, ld_pk, wq, wk, pos, grid_H, grid_W, tps, block, \
                                    bps, n_blocks, rope, n_tokens, n_heads, eps, s);
        SOL_POOL_STAGE_U(1) SOL_POOL_STAGE_U(2) SOL_POOL_STAGE_U(3) SOL_POOL_STAGE_U(4) SOL_POOL_STAGE_U(5)
        SOL_POOL_STAGE_U(6)
#undef SOL_POOL_STAGE_U
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
