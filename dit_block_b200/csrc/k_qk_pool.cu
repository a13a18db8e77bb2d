// k_qk_pool.cu -- the QKV epilogue (QK RMSNorm + 3D RoPE, in place) fused with the
// block means that SubBlock sparse attention routes on ["8xH200 上的 MiniMax-H3"
// (xhh.club), Q&A on SubBlock: the sequence is cut into 64-token blocks and a router
// keeps a fraction of the key blocks; "SGLang acelera video do MiniMax-H3",
// "De onde vem os ganhos"].
//
// bf16 with head_dim 128 and an even number of heads up to 48 takes the staged kernel
// k_qk_pool_stage (k_qk_cta.cu: a ring of bulk-copied rows per block, 6.27-6.41 TB/s at
// 245,952 tokens x 40 heads, where a row-in-registers kernel that walked each block two
// tokens at a time reached 6.08).  Every other shape takes k_qk_rope_pool:
// a CTA of 8 warps owns one block of `block` tokens at a time (blocks restart at every
// sample boundary; blocks walked with a grid stride).  Each warp takes a contiguous run
// of the block's tokens and walks it in chunks of up to 8 tokens: it first stages the
// chunk's (cos, sin) pairs in shared memory, then for every head-vector step (16 lanes
// per vector, as in the plain epilogue) loads that vector of all the chunk's tokens (8
// loads in flight per lane), normalises and rotates each, stores it in place, and sums
// the chunk in registers, adding the sum into a per-CTA fp32 accumulator in shared
// memory once per chunk (a padded layout keeps the two head vectors of a warp step on
// different banks).  After the block, one barrier; the CTA scales the sums by 1/count,
// stores the pooled q and k rows and clears the accumulator.  Means are taken over the
// fp32 results before their rounding to the output type.

#include <atomic>

#include "common.cuh"
#include "launch.h"

namespace sol {

constexpr int kPoolWarps = 8;
constexpr size_t kPoolSmemMax = 110 * 1024;  // accumulator of one CTA, at most

// Shared-memory accumulator layout: vector vi, element e of lane slot `sub` at
// vi * (HD + 16) + e * LPH + sub.  Lanes of one head vector hit consecutive words and
// the +16 pad puts the second vector of a warp step on the other 16 banks.
template <int LPH, int E>
__device__ __forceinline__ int acc_index(int vi, int e, int sub)
{
    return vi * (LPH * E + 16) + e * LPH + sub;
}

constexpr int kChunk = 8;  // tokens a warp handles together per head-vector step

template <typename T, int LPH>
__global__ void __launch_bounds__(32 * kPoolWarps)
k_qk_rope_pool(T* q, T* k, int64_t ld_q, int64_t ld_k, T* pq, T* pk, int64_t ld_pq, int64_t ld_pk,
               const T* __restrict__ wq, const T* __restrict__ wk, const int32_t* __restrict__ pos,
               int32_t grid_H, int32_t grid_W, int64_t tps, int32_t block, int64_t blocks_per_sample,
               int64_t n_blocks, RopeDev rope, int64_t n_tokens, int32_t n_heads, float eps)
{
    constexpr int E = Vec<T>::N;
    constexpr int P = E / 2;
    constexpr int HPW = 32 / LPH;
    constexpr int HD = LPH * E;
    constexpr int NPAIR = HD / 2;
    extern __shared__ __align__(16) float smem_f[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int sub = lane % LPH;
    const int grp = lane / LPH;
    const int n_vec = 2 * n_heads;
    const int steps = (n_vec + HPW - 1) / HPW;
    const int acc_len = n_vec * (HD + 16);
    float* acc_s = smem_f;
    // per warp: the (cos, sin) of every pair of its current chunk of tokens
    float2* cs_s = reinterpret_cast<float2*>(smem_f + acc_len) + warp * kChunk * NPAIR;

    const uint4 wq_raw = wq ? ld_cached(wq + sub * E) : make_uint4(0u, 0u, 0u, 0u);
    const uint4 wk_raw = wk ? ld_cached(wk + sub * E) : make_uint4(0u, 0u, 0u, 0u);
    const float2* tab0 = rope.tab[0];
    int tidx[P], stride[P], axis[P];
#pragma unroll
    for (int m = 0; m < P; ++m) {
        const int pi = sub * P + m;
        const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
        axis[m] = pi < h0 ? 0 : (pi < h01 ? 1 : 2);
        const float2* t = axis[m] == 0 ? rope.tab[0] + pi
                                       : (axis[m] == 1 ? rope.tab[1] + (pi - h0) : rope.tab[2] + (pi - h01));
        tidx[m] = (int)(t - tab0);
        stride[m] = axis[m] == 0 ? rope.half[0] : (axis[m] == 1 ? rope.half[1] : rope.half[2]);
    }

    for (int i = threadIdx.x; i < acc_len; i += blockDim.x) acc_s[i] = 0.f;
    __syncthreads();

    for (int64_t blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const int64_t sample = blk / blocks_per_sample;
        const int64_t t0 = sample * tps + (blk - sample * blocks_per_sample) * block;
        int64_t t1 = t0 + block;
        if (t1 > (sample + 1) * tps) t1 = (sample + 1) * tps;
        if (t1 > n_tokens) t1 = n_tokens;
        const int64_t per_warp = (t1 - t0 + kPoolWarps - 1) / kPoolWarps;
        const int64_t w0 = t0 + warp * per_warp;
        const int64_t w1 = w0 + per_warp < t1 ? w0 + per_warp : t1;
        int g0 = 0, g1 = 0, g2 = 0;
        if (!pos && w0 < w1) {
            const int64_t nl = w0 - sample * tps;
            g0 = (int)(nl / ((int64_t)grid_H * grid_W));
            g1 = (int)((nl / grid_W) % grid_H);
            g2 = (int)(nl % grid_W);
        }
        for (int64_t c0 = w0; c0 < w1; c0 += kChunk) {
            const int cn = (int)(w1 - c0 < kChunk ? w1 - c0 : kChunk);  // tokens in this chunk
            // (cos, sin) of this lane's pairs for each token of the chunk
            for (int t = 0; t < cn; ++t) {
                const int64_t n = c0 + t;
                int p0, p1, p2;
                if (pos) {
                    p0 = min(max(__ldg(pos + 3 * n + 0), 0), rope.max[0] - 1);
                    p1 = min(max(__ldg(pos + 3 * n + 1), 0), rope.max[1] - 1);
                    p2 = min(max(__ldg(pos + 3 * n + 2), 0), rope.max[2] - 1);
                } else {
                    p0 = g0;
                    p1 = g1;
                    p2 = g2;
                    if (++g2 == grid_W) {
                        g2 = 0;
                        if (++g1 == grid_H) {
                            g1 = 0;
                            ++g0;
                        }
                    }
                }
                if (grp == 0) {
#pragma unroll
                    for (int m = 0; m < P; ++m) {
                        const int pm = axis[m] == 0 ? p0 : (axis[m] == 1 ? p1 : p2);
                        cs_s[t * NPAIR + sub * P + m] = __ldg(tab0 + tidx[m] + (int64_t)pm * stride[m]);
                    }
                }
            }
            __syncwarp();
            for (int st = 0; st < steps; ++st) {
                const int vi = st * HPW + grp;
                const bool is_q = vi < n_heads;
                const bool valid = vi < n_vec;
                const T* src = is_q ? q + (int64_t)vi * HD : k + (int64_t)(vi - n_heads) * HD;
                const int64_t ld = is_q ? ld_q : ld_k;
                uint4 raw[kChunk];
#pragma unroll
                for (int t = 0; t < kChunk; ++t)
                    raw[t] = (t < cn && valid) ? ld_stream(src + (c0 + t) * ld + sub * E)
                                               : make_uint4(0u, 0u, 0u, 0u);
                float w[E];
                if ((is_q ? wq : wk) != nullptr) {
                    unpack<T>(is_q ? wq_raw : wk_raw, w);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) w[e] = 1.f;
                }
                float acc[E];
#pragma unroll
                for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
                for (int t = 0; t < kChunk; ++t) {
                    if (t >= cn) break;  // uniform across the warp
                    float f[E];
                    unpack<T>(raw[t], f);
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
                    for (int off = LPH / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    const float r = rsqrtf(ss * (1.f / HD) + eps);
                    float o[E];
#pragma unroll
                    for (int m = 0; m < P; ++m) {
                        const float2 c = cs_s[t * NPAIR + sub * P + m];
                        const float a = f[2 * m] * r * w[2 * m];
                        const float b = f[2 * m + 1] * r * w[2 * m + 1];
                        o[2 * m] = a * c.x - b * c.y;
                        o[2 * m + 1] = a * c.y + b * c.x;
                    }
#pragma unroll
                    for (int e = 0; e < E; ++e) acc[e] += o[e];
                    if (valid) st_stream(const_cast<T*>(src) + (c0 + t) * ld + sub * E, pack<T>(o));
                }
                if (valid) {
#pragma unroll
                    for (int e = 0; e < E; ++e) atomicAdd(&acc_s[acc_index<LPH, E>(vi, e, sub)], acc[e]);
                }
            }
            __syncwarp();  // the (cos, sin) cache is rewritten by the next chunk
        }
        __syncthreads();
        // block mean: each thread finishes 16-byte slices of the pooled rows and clears them
        const float inv = 1.f / (float)(t1 - t0);
        for (int c = threadIdx.x; c < n_vec * LPH; c += blockDim.x) {
            const int vi = c / LPH, sl = c % LPH;
            float o[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float* a = &acc_s[acc_index<LPH, E>(vi, e, sl)];
                o[e] = *a * inv;
                *a = 0.f;
            }
            if (vi < n_heads)
                st_stream(pq + blk * ld_pq + (int64_t)vi * HD + sl * E, pack<T>(o));
            else
                st_stream(pk + blk * ld_pk + (int64_t)(vi - n_heads) * HD + sl * E, pack<T>(o));
        }
        __syncthreads();
    }
}

namespace {

constexpr int kPoolThreads = 32 * kPoolWarps;

template <typename T, int LPH>
cudaError_t run_pool(void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk, int64_t ld_pq,
                     int64_t ld_pk, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                     int32_t grid_W, int64_t tps, int32_t block, int64_t bps, int64_t n_blocks,
                     const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    const void* kfn = (const void*)k_qk_rope_pool<T, LPH>;
    const size_t smem = qk_pool_smem_bytes(sizeof(T) == 2 ? SOL_DTYPE_BF16 : SOL_DTYPE_F32, n_heads,
                                           LPH * Vec<T>::N);
    static std::atomic<bool> attr_set[64];  // per device; a repeated set is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        const cudaError_t e =
            cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPoolSmemMax);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    int64_t grid = (int64_t)ctas_per_sm(kfn, kPoolThreads, smem) * sm_count();
    if (grid > n_blocks) grid = n_blocks;
    if (grid < 1) grid = 1;
    k_qk_rope_pool<T, LPH><<<(unsigned)grid, kPoolThreads, smem, s>>>(
        (T*)q, (T*)k, ld_q, ld_k, (T*)pq, (T*)pk, ld_pq, ld_pk, (const T*)wq, (const T*)wk, pos, grid_H,
        grid_W, tps, block, bps, n_blocks, rope, n_tokens, n_heads, eps);
    return cudaGetLastError();
}

}  // namespace

size_t qk_pool_smem_bytes(sol_dtype dt, int32_t n_heads, int32_t head_dim)
{
    (void)dt;
    const size_t acc = (size_t)2 * (size_t)n_heads * (size_t)(head_dim + 16) * sizeof(float);
    const size_t cs = (size_t)kPoolWarps * kChunk * (size_t)(head_dim / 2) * sizeof(float2);
    return acc + cs;
}

size_t qk_pool_smem_limit() { return kPoolSmemMax; }

cudaError_t launch_qk_rope_pool(sol_dtype dt, void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq,
                                void* pk, int64_t ld_pq, int64_t ld_pk, const void* wq, const void* wk,
                                const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps,
                                int32_t block, int64_t bps, int64_t n_blocks, const RopeDev& rope,
                                int64_t n_tokens, int32_t n_heads, int32_t head_dim, float eps,
                                cudaStream_t s)
{
    if (qk_pool_stage_fits(dt, n_heads, head_dim, q, k, tps, n_blocks))  // staged rows (k_qk_cta.cu)
        return launch_qk_pool_stage(q, k, ld_q, ld_k, pq, pk, ld_pq, ld_pk, wq, wk, pos, grid_H, grid_W, tps, block,
                                    bps, n_blocks, rope, n_tokens, n_heads, eps, s);
    const int lph = head_dim / (dt == SOL_DTYPE_BF16 ? 8 : 4);
#define ARGS q, k, ld_q, ld_k, pq, pk, ld_pq, ld_pk, wq, wk, pos, grid_H, grid_W, tps, block, bps, n_blocks, rope, n_tokens, n_heads, eps, s
    if (dt == SOL_DTYPE_BF16) {
        switch (lph) {
        case 8: return run_pool<bf16, 8>(ARGS);
        case 16: return run_pool<bf16, 16>(ARGS);
        case 32: return run_pool<bf16, 32>(ARGS);
        default: return cudaErrorInvalidConfiguration;
        }
    }
    switch (lph) {
    case 8: return run_pool<float, 8>(ARGS);
    case 16: return run_pool<float, 16>(ARGS);
    case 32: return run_pool<float, 32>(ARGS);
    default: return cudaErrorInvalidConfiguration;
    }
#undef ARGS
}

}  // namespace sol
