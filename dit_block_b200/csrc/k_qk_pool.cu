// k_qk_pool.cu -- the QKV epilogue (QK RMSNorm + 3D RoPE, in place) fused with the
// block means that SubBlock sparse attention routes on ["8xH200 上的 MiniMax-H3"
// (xhh.club), Q&A on SubBlock: the sequence is cut into 64-token blocks and a router
// keeps a fraction of the key blocks; "SGLang acelera video do MiniMax-H3",
// "De onde vem os ganhos"].
//
// One CTA (16 warps) per block of `block` tokens (blocks restart at every sample
// boundary), blocks walked with a grid stride.  Warps are assigned to head vectors, not
// to tokens.  Warp w
// owns steps w, w + nwarps, ... of the token's 2*n_heads head vectors (q heads, then k
// heads; a step is 32/LPH vectors, one per lane group), walks all tokens of the block
// and keeps its lanes' slices of those vectors' running sums in registers.  So the block
// mean needs no cross-warp reduction: after the block's last token each lane scales its
// sums by 1/count and stores its slice of the pooled q and k rows.  The per-token work
// is the epilogue's: RMS over the LPH lanes of a vector, weights, rotation by the
// token's (cos, sin) from the fp32 tables, store in place.  Means are taken over the
// fp32 results before their rounding to the output type.
#include "common.cuh"
#include "launch.h"

namespace sol {

template <typename T, int LPH, int MAXV>
__global__ void __launch_bounds__(512, 1)
k_qk_rope_pool(T* q, T* k, int64_t ld_q, int64_t ld_k, T* pq, T* pk, int64_t ld_pq, int64_t ld_pk,
               const T* __restrict__ wq, const T* __restrict__ wk, const int32_t* __restrict__ pos,
               int32_t grid_H, int32_t grid_W, int64_t tps, int32_t block, int64_t blocks_per_sample,
               int64_t n_blocks, RopeDev rope, int64_t n_tokens, int32_t n_heads, float eps)
{
    constexpr int E = Vec<T>::N;
    constexpr int P = E / 2;
    constexpr int HPW = 32 / LPH;
    constexpr int HD = LPH * E;
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPH;
    const int grp = lane / LPH;
    const int warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int n_vec = 2 * n_heads;
    const int steps = (n_vec + HPW - 1) / HPW;

    // weights kept packed (widened per use) and table entries as 32-bit indices into the
    // one allocation holding the three axis tables: fewer live registers
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

    for (int64_t blk = blockIdx.x; blk < n_blocks; blk += gridDim.x) {
        const int64_t sample = blk / blocks_per_sample;
        const int64_t t0 = sample * tps + (blk - sample * blocks_per_sample) * block;
        int64_t t1 = t0 + block;
        if (t1 > (sample + 1) * tps) t1 = (sample + 1) * tps;
        if (t1 > n_tokens) t1 = n_tokens;

        float acc[MAXV][E];
#pragma unroll
        for (int v = 0; v < MAXV; ++v)
#pragma unroll
            for (int e = 0; e < E; ++e) acc[v][e] = 0.f;

        for (int64_t n = t0; n < t1; ++n) {
            int p0, p1, p2;
            if (pos) {
                p0 = min(max(__ldg(pos + 3 * n + 0), 0), rope.max[0] - 1);
                p1 = min(max(__ldg(pos + 3 * n + 1), 0), rope.max[1] - 1);
                p2 = min(max(__ldg(pos + 3 * n + 2), 0), rope.max[2] - 1);
            } else {
                const int64_t nl = n - sample * tps;
                p0 = (int)(nl / ((int64_t)grid_H * grid_W));
                p1 = (int)((nl / grid_W) % grid_H);
                p2 = (int)(nl % grid_W);
            }
            uint4 raw[MAXV];
#pragma unroll
            for (int v = 0; v < MAXV; ++v) {
                const int vi = (warp + v * nwarps) * HPW + grp;
                if (vi < n_heads)
                    raw[v] = ld_stream(q + n * ld_q + (int64_t)vi * HD + sub * E);
                else if (vi < n_vec)
                    raw[v] = ld_stream(k + n * ld_k + (int64_t)(vi - n_heads) * HD + sub * E);
                else
                    raw[v] = make_uint4(0u, 0u, 0u, 0u);
            }
            float cs[P], sn[P];
#pragma unroll
            for (int m = 0; m < P; ++m) {
                const int pm = axis[m] == 0 ? p0 : (axis[m] == 1 ? p1 : p2);
                const float2 t = __ldg(tab0 + tidx[m] + (int64_t)pm * stride[m]);
                cs[m] = t.x;
                sn[m] = t.y;
            }
#pragma unroll
            for (int v = 0; v < MAXV; ++v) {
                const int step = warp + v * nwarps;
                if (step >= steps) break;  // uniform across the warp
                const int vi = step * HPW + grp;
                float f[E];
                unpack<T>(raw[v], f);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
                for (int off = LPH / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float r = rsqrtf(ss * (1.f / HD) + eps);
                const bool is_q = vi < n_heads;
                float w[E];
                if ((is_q ? wq : wk) != nullptr) {
                    unpack<T>(is_q ? wq_raw : wk_raw, w);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) w[e] = 1.f;
                }
                float o[E];
#pragma unroll
                for (int m = 0; m < P; ++m) {
                    const float a = f[2 * m] * r * w[2 * m];
                    const float b = f[2 * m + 1] * r * w[2 * m + 1];
                    o[2 * m] = a * cs[m] - b * sn[m];
                    o[2 * m + 1] = a * sn[m] + b * cs[m];
                }
#pragma unroll
                for (int e = 0; e < E; ++e) acc[v][e] += o[e];
                if (is_q)
                    st_stream(q + n * ld_q + (int64_t)vi * HD + sub * E, pack<T>(o));
                else if (vi < n_vec)
                    st_stream(k + n * ld_k + (int64_t)(vi - n_heads) * HD + sub * E, pack<T>(o));
            }
        }

        const float inv = 1.f / (float)(t1 - t0);
#pragma unroll
        for (int v = 0; v < MAXV; ++v) {
            const int step = warp + v * nwarps;
            const int vi = step * HPW + grp;
            if (step >= steps || vi >= n_vec) continue;
            float o[E];
#pragma unroll
            for (int e = 0; e < E; ++e) o[e] = acc[v][e] * inv;
            if (vi < n_heads)
                st_stream(pq + blk * ld_pq + (int64_t)vi * HD + sub * E, pack<T>(o));
            else
                st_stream(pk + blk * ld_pk + (int64_t)(vi - n_heads) * HD + sub * E, pack<T>(o));
        }
    }
}

namespace {

constexpr int kPoolThreads = 512;

template <typename T, int LPH, int MAXV>
cudaError_t run_pool(void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk, int64_t ld_pq,
                     int64_t ld_pk, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                     int32_t grid_W, int64_t tps, int32_t block, int64_t bps, int64_t n_blocks,
                     const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
    const void* kfn = (const void*)k_qk_rope_pool<T, LPH, MAXV>;
    int64_t grid = (int64_t)ctas_per_sm(kfn, kPoolThreads, 0) * sm_count();
    if (grid > n_blocks) grid = n_blocks;
    if (grid < 1) grid = 1;
    k_qk_rope_pool<T, LPH, MAXV><<<(unsigned)grid, kPoolThreads, 0, s>>>(
        (T*)q, (T*)k, ld_q, ld_k, (T*)pq, (T*)pk, ld_pq, ld_pk, (const T*)wq, (const T*)wk, pos, grid_H,
        grid_W, tps, block, bps, n_blocks, rope, n_tokens, n_heads, eps);
    return cudaGetLastError();
}

template <typename T, int LPH>
cudaError_t dispatch_maxv(int vpl, void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk,
                          int64_t ld_pq, int64_t ld_pk, const void* wq, const void* wk,
                          const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps, int32_t block,
                          int64_t bps, int64_t n_blocks, const RopeDev& rope, int64_t n_tokens,
                          int32_t n_heads, float eps, cudaStream_t s)
{
#define ARGS q, k, ld_q, ld_k, pq, pk, ld_pq, ld_pk, wq, wk, pos, grid_H, grid_W, tps, block, bps, n_blocks, rope, n_tokens, n_heads, eps, s
    if (vpl <= 1) return run_pool<T, LPH, 1>(ARGS);
    if (vpl <= 2) return run_pool<T, LPH, 2>(ARGS);
    if (vpl <= 3) return run_pool<T, LPH, 3>(ARGS);
    if (vpl <= 5) return run_pool<T, LPH, 5>(ARGS);
    return cudaErrorInvalidConfiguration;
#undef ARGS
}

}  // namespace

int qk_pool_max_vectors_per_lane() { return 5; }

int qk_pool_vectors_per_lane(sol_dtype dt, int32_t n_heads, int32_t head_dim)
{
    const int lph = head_dim / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const int hpw = 32 / lph;
    const int steps = (2 * n_heads + hpw - 1) / hpw;
    const int nwarps = kPoolThreads / 32;
    return (steps + nwarps - 1) / nwarps;
}

cudaError_t launch_qk_rope_pool(sol_dtype dt, void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq,
                                void* pk, int64_t ld_pq, int64_t ld_pk, const void* wq, const void* wk,
                                const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps,
                                int32_t block, int64_t bps, int64_t n_blocks, const RopeDev& rope,
                                int64_t n_tokens, int32_t n_heads, int32_t head_dim, float eps,
                                cudaStream_t s)
{
    const int vpl = qk_pool_vectors_per_lane(dt, n_heads, head_dim);
    const int lph = head_dim / (dt == SOL_DTYPE_BF16 ? 8 : 4);
#define ARGS vpl, q, k, ld_q, ld_k, pq, pk, ld_pq, ld_pk, wq, wk, pos, grid_H, grid_W, tps, block, bps, n_blocks, rope, n_tokens, n_heads, eps, s
    if (dt == SOL_DTYPE_BF16) {
        switch (lph) {
        case 8: return dispatch_maxv<bf16, 8>(ARGS);
        case 16: return dispatch_maxv<bf16, 16>(ARGS);
        case 32: return dispatch_maxv<bf16, 32>(ARGS);
        default: return cudaErrorInvalidConfiguration;
        }
    }
    switch (lph) {
    case 8: return dispatch_maxv<float, 8>(ARGS);
    case 16: return dispatch_maxv<float, 16>(ARGS);
    case 32: return dispatch_maxv<float, 32>(ARGS);
    default: return cudaErrorInvalidConfiguration;
    }
#undef ARGS
}

}  // namespace sol
