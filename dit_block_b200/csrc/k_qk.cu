// k_qk.cu -- QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合"], and
// through it the QKV-projection epilogue.
//
// One warp per token, tokens walked with a grid stride.  A head vector is LPH lanes x
// one 16-byte vector each (bf16 head_dim 128: 16 lanes x 8 elements), so a warp covers
// 32/LPH head vectors per step and walks the token's 2*n_heads vectors (q heads, then
// k heads).  A lane always owns the same element slice of every head vector, so:
//   * its RMSNorm weights (wq and wk slices) are loaded once per thread;
//   * its rotary pairs always belong to the same (axis, frequency) entries, so per
//     token it fetches just E/2 (cos, sin) pairs from the L1-resident table and reuses
//     them for all 2*n_heads vectors;
//   * the RMS reduction is an xor-shuffle tree over the LPH lanes of one vector.
// UNR head-vector loads are issued before any is used to keep HBM busy.  Each lane
// reads and then writes only its own 16 bytes, so in-place operation is safe.
#include "common.cuh"
#include "launch.h"

namespace sol {

template <typename T, int LPH, int UNR>
__global__ void __launch_bounds__(256)
k_qk_rmsnorm_rope3d(T* q_out, T* k_out, int64_t ld_qo, int64_t ld_ko, const T* q, const T* k,
                    int64_t ld_q, int64_t ld_k, const T* __restrict__ wq,
                    const T* __restrict__ wk, const int32_t* __restrict__ pos, int32_t grid_H,
                    int32_t grid_W, int64_t tokens_per_sample, RopeDev rope, int64_t n_tokens,
                    int32_t n_heads, float eps)
{
    constexpr int E = Vec<T>::N;   // elements per lane per head vector
    constexpr int P = E / 2;       // rotary pairs per lane
    constexpr int HPW = 32 / LPH;  // head vectors per warp step
    constexpr int HD = LPH * E;    // head_dim
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPH;
    const int grp = lane / LPH;

    float fwq[E], fwk[E];
    if (wq) {
        unpack<T>(ld_cached(wq + sub * E), fwq);
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) fwq[e] = 1.f;
    }
    if (wk) {
        unpack<T>(ld_cached(wk + sub * E), fwk);
    } else {
#pragma unroll
        for (int e = 0; e < E; ++e) fwk[e] = 1.f;
    }

    // Table entry base and row stride of each of this lane's pairs; the position axis
    // is picked with selects (no dynamic indexing, so nothing spills to local memory).
    const float2* tb[P];
    int stride[P], axis[P];
#pragma unroll
    for (int m = 0; m < P; ++m) {
        const int pi = sub * P + m;
        const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
        axis[m] = pi < h0 ? 0 : (pi < h01 ? 1 : 2);
        tb[m] = axis[m] == 0 ? rope.tab[0] + pi : (axis[m] == 1 ? rope.tab[1] + (pi - h0) : rope.tab[2] + (pi - h01));
        stride[m] = axis[m] == 0 ? rope.half[0] : (axis[m] == 1 ? rope.half[1] : rope.half[2]);
    }

    const int n_vec = 2 * n_heads;
    const int steps = (n_vec + HPW - 1) / HPW;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warp_step = ((int64_t)gridDim.x * blockDim.x) >> 5;

    for (int64_t n = warp0; n < n_tokens; n += warp_step) {
        int p0, p1, p2;
        if (pos) {
            p0 = min(max(__ldg(pos + 3 * n + 0), 0), rope.max[0] - 1);
            p1 = min(max(__ldg(pos + 3 * n + 1), 0), rope.max[1] - 1);
            p2 = min(max(__ldg(pos + 3 * n + 2), 0), rope.max[2] - 1);
        } else {
            const int64_t nl = tokens_per_sample > 0 ? n % tokens_per_sample : n;
            p0 = (int)(nl / ((int64_t)grid_H * grid_W));
            p1 = (int)((nl / grid_W) % grid_H);
            p2 = (int)(nl % grid_W);
        }
        float cs[P], sn[P];
#pragma unroll
        for (int m = 0; m < P; ++m) {
            const int pm = axis[m] == 0 ? p0 : (axis[m] == 1 ? p1 : p2);
            const float2 t = __ldg(tb[m] + (int64_t)pm * stride[m]);
            cs[m] = t.x;
            sn[m] = t.y;
        }

        for (int s0 = 0; s0 < steps; s0 += UNR) {
            uint4 raw[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int vi = (s0 + u) * HPW + grp;
                if (vi < n_heads)
                    raw[u] = ld_stream(q + n * ld_q + (int64_t)vi * HD + sub * E);
                else if (vi < n_vec)
                    raw[u] = ld_stream(k + n * ld_k + (int64_t)(vi - n_heads) * HD + sub * E);
                else
                    raw[u] = make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int vi = (s0 + u) * HPW + grp;
                float f[E];
                unpack<T>(raw[u], f);
                float ss = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
                for (int off = LPH / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                const float r = rsqrtf(ss * (1.f / HD) + eps);
                const bool is_q = vi < n_heads;
                float o[E];
#pragma unroll
                for (int m = 0; m < P; ++m) {
                    const float a = f[2 * m] * r * (is_q ? fwq[2 * m] : fwk[2 * m]);
                    const float b = f[2 * m + 1] * r * (is_q ? fwq[2 * m + 1] : fwk[2 * m + 1]);
                    o[2 * m] = a * cs[m] - b * sn[m];
                    o[2 * m + 1] = a * sn[m] + b * cs[m];
                }
                if (is_q)
                    st_stream(q_out + n * ld_qo + (int64_t)vi * HD + sub * E, pack<T>(o));
                else if (vi < n_vec)
                    st_stream(k_out + n * ld_ko + (int64_t)(vi - n_heads) * HD + sub * E, pack<T>(o));
            }
        }
    }
}

namespace {

constexpr int kQkThreads = 256;

template <typename T, int LPH>
cudaError_t run_qk(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q,
                   const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk,
                   const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps,
                   const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps,
                   cudaStream_t s)
{
    constexpr int UNR = 8;
    const void* kfn = (const void*)k_qk_rmsnorm_rope3d<T, LPH, UNR>;
    const int64_t warps_needed = n_tokens;
    int64_t grid = (int64_t)ctas_per_sm(kfn, kQkThreads, 0) * sm_count();
    const int64_t max_grid = (warps_needed + (kQkThreads / 32) - 1) / (kQkThreads / 32);
    if (grid > max_grid) grid = max_grid;
    if (grid < 1) grid = 1;
    k_qk_rmsnorm_rope3d<T, LPH, UNR><<<(unsigned)grid, kQkThreads, 0, s>>>(
        (T*)q_out, (T*)k_out, ld_qo, ld_ko, (const T*)q, (const T*)k, ld_q, ld_k, (const T*)wq,
        (const T*)wk, pos, grid_H, grid_W, tps, rope, n_tokens, n_heads, eps);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qk_rmsnorm_rope3d(sol_dtype dt, void* q_out, void* k_out, int64_t ld_qo,
                                     int64_t ld_ko, const void* q, const void* k, int64_t ld_q,
                                     int64_t ld_k, const void* wq, const void* wk,
                                     const int32_t* pos, int32_t grid_T, int32_t grid_H,
                                     int32_t grid_W, int64_t tps, const RopeDev& rope,
                                     int64_t n_tokens, int32_t n_heads, int32_t head_dim,
                                     float eps, cudaStream_t s)
{
    (void)grid_T;
    if (qk_cta_fits(dt, n_heads, head_dim, q, k, n_tokens))
        return launch_qk_cta(q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope,
                             n_tokens, n_heads, eps, s);
    if (qk_regs_fits(dt, n_heads, head_dim))
        return launch_qk_regs(q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope,
                              n_tokens, n_heads, eps, s);
    const int E = dt == SOL_DTYPE_BF16 ? 8 : 4;
    const int lph = head_dim / E;
#define ARGS q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, n_tokens, n_heads, eps, s
    if (dt == SOL_DTYPE_BF16) {
        switch (lph) {
        case 8: return run_qk<bf16, 8>(ARGS);
        case 16: return run_qk<bf16, 16>(ARGS);
        case 32: return run_qk<bf16, 32>(ARGS);
        default: return cudaErrorInvalidConfiguration;
        }
    }
    switch (lph) {
    case 8: return run_qk<float, 8>(ARGS);
    case 16: return run_qk<float, 16>(ARGS);
    case 32: return run_qk<float, 32>(ARGS);
    default: return cudaErrorInvalidConfiguration;
    }
#undef ARGS
}

}  // namespace sol
