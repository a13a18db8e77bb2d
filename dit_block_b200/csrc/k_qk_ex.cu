// k_qk_ex.cu -- QK RMSNorm + 3D RoPE in the convention variants the pages leave open:
// the norm over each head vector or over all heads of the row, interleaved or rotate-half
// rotary pairs, and outputs at any (token, head, sample) strides -- e.g. straight into an
// attention-friendly [sample, head, token, dim] layout.
//
// Same mapping as k_qk.cu: one warp per token, LPH lanes x one 16-byte vector per head
// vector, per-lane weights (or, across heads, one 16-byte weight slice per vector) and
// per-token (cos, sin) reused over the token's vectors.
//   ACROSS (norm over all heads): a first pass over the token's q and k vectors sums
//     both squares with full-warp shuffles; the second pass re-reads the row (an L2 hit:
//     it was read a moment before) to normalise, rotate and store.
//   HALF (rotate-half pairs): element j of an axis chunk pairs with element j + D_c/2.
//     A lane's E elements sit in one half of one chunk (chunk widths are multiples of
//     2E), so its partners all live in lane +-(D_c/2)/E of the same head vector: one
//     shuffle per element brings them over.
#include "common.cuh"
#include "launch.h"

namespace sol {

template <typename T, int LPH, int UNR, bool ACROSS, bool HALF>
__global__ void __launch_bounds__(256)
k_qk_ex(T* q_out, T* k_out, QkOutStrides os, const T* q, const T* k, int64_t ld_q, int64_t ld_k,
        const T* __restrict__ wq, const T* __restrict__ wk, const int32_t* __restrict__ pos,
        int32_t grid_H, int32_t grid_W, int64_t tps, RopeDev rope, int64_t n_tokens, int32_t n_heads,
        float eps)
{
    constexpr int E = Vec<T>::N;
    constexpr int P = E / 2;
    constexpr int HPW = 32 / LPH;
    constexpr int HD = LPH * E;
    constexpr int NT = HALF ? E : P;  // (cos, sin) entries per lane per token
    const int lane = threadIdx.x & 31;
    const int sub = lane % LPH;
    const int grp = lane / LPH;
    const int n_vec = 2 * n_heads;
    const int steps = (n_vec + HPW - 1) / HPW;

    // per-head weights live in registers; across heads they are read per vector
    float fwq[E], fwk[E];
#pragma unroll
    for (int e = 0; e < E; ++e) fwq[e] = fwk[e] = 1.f;
    if (!ACROSS) {
        if (wq) unpack<T>(ld_cached(wq + sub * E), fwq);
        if (wk) unpack<T>(ld_cached(wk + sub * E), fwk);
    }

    // table entries of this lane: interleaved -> its P pairs; rotate-half -> one entry per
    // element (frequency j of the element inside its chunk half)
    const float2* tab0 = rope.tab[0];
    int tidx[NT], stride[NT], axis[NT];
    int partner = lane;
    float sgn = 1.f;
#pragma unroll
    for (int m = 0; m < NT; ++m) {
        const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
        int ax, j;
        if (HALF) {
            const int i = sub * E + m;  // element index inside the head vector
            const int c0 = 2 * h0, c1 = 2 * h01;
            ax = i < c0 ? 0 : (i < c1 ? 1 : 2);
            const int off = ax == 0 ? 0 : (ax == 1 ? c0 : c1);
            const int hw = rope.half[ax];
            j = (i - off) % hw;
            if (m == 0) {  // every element of the lane lies in the same chunk half
                const int d_lanes = hw / E;
                const bool first = (i - off) < hw;
                partner = first ? lane + d_lanes : lane - d_lanes;
                sgn = first ? -1.f : 1.f;
            }
        } else {
            const int pi = sub * P + m;
            ax = pi < h0 ? 0 : (pi < h01 ? 1 : 2);
            j = ax == 0 ? pi : (ax == 1 ? pi - h0 : pi - h01);
        }
        axis[m] = ax;
        tidx[m] = (int)(rope.tab[ax] - tab0) + j;
        stride[m] = rope.half[ax];
    }

    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t warp_step = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t n = warp0; n < n_tokens; n += warp_step) {
        const int64_t sample = tps > 0 ? n / tps : 0;
        const int64_t nl = n - sample * tps;
        int p0, p1, p2;
        if (pos) {
            p0 = min(max(__ldg(pos + 3 * n + 0), 0), rope.max[0] - 1);
            p1 = min(max(__ldg(pos + 3 * n + 1), 0), rope.max[1] - 1);
            p2 = min(max(__ldg(pos + 3 * n + 2), 0), rope.max[2] - 1);
        } else {
            p0 = (int)(nl / ((int64_t)grid_H * grid_W));
            p1 = (int)((nl / grid_W) % grid_H);
            p2 = (int)(nl % grid_W);
        }
        float cs[NT], sn[NT];
#pragma unroll
        for (int m = 0; m < NT; ++m) {
            const int pm = axis[m] == 0 ? p0 : (axis[m] == 1 ? p1 : p2);
            const float2 t = __ldg(tab0 + tidx[m] + (int64_t)pm * stride[m]);
            cs[m] = t.x;
            sn[m] = t.y;
        }
        const T* qrow = q + n * ld_q;
        const T* krow = k + n * ld_k;
        T* qo = q_out + sample * os.sample + nl * os.token;
        T* ko = k_out + sample * os.sample + nl * os.token;

        float rq = 0.f, rk = 0.f;
        if (ACROSS) {
            float sq = 0.f, sk = 0.f;
            for (int s0 = 0; s0 < steps; s0 += UNR) {
                uint4 raw[UNR];
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int vi = (s0 + u) * HPW + grp;
                    raw[u] = vi < n_heads ? ld_plain(qrow + (int64_t)vi * HD + sub * E)
                                          : (vi < n_vec ? ld_plain(krow + (int64_t)(vi - n_heads) * HD + sub * E)
                                                        : make_uint4(0u, 0u, 0u, 0u));
                }
#pragma unroll
                for (int u = 0; u < UNR; ++u) {
                    const int vi = (s0 + u) * HPW + grp;
                    float f[E];
                    unpack<T>(raw[u], f);
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
                    if (vi < n_heads) sq += ss; else sk += ss;
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                sq += __shfl_xor_sync(0xffffffffu, sq, off);
                sk += __shfl_xor_sync(0xffffffffu, sk, off);
            }
            const float inv_n = 1.f / ((float)n_heads * HD);
            rq = rsqrtf(sq * inv_n + eps);
            rk = rsqrtf(sk * inv_n + eps);
        }

        for (int s0 = 0; s0 < steps; s0 += UNR) {
            uint4 raw[UNR];
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int vi = (s0 + u) * HPW + grp;
                raw[u] = vi < n_heads ? ld_stream(qrow + (int64_t)vi * HD + sub * E)
                                      : (vi < n_vec ? ld_stream(krow + (int64_t)(vi - n_heads) * HD + sub * E)
                                                    : make_uint4(0u, 0u, 0u, 0u));
            }
#pragma unroll
            for (int u = 0; u < UNR; ++u) {
                const int vi = (s0 + u) * HPW + grp;
                const bool is_q = vi < n_heads;
                float f[E];
                unpack<T>(raw[u], f);
                float r;
                float w[E];
                if (ACROSS) {
                    r = is_q ? rq : rk;
                    const T* wsrc = is_q ? wq : wk;
                    const int h = is_q ? vi : vi - n_heads;
                    if (wsrc && vi < n_vec) {
                        unpack<T>(ld_cached(wsrc + (int64_t)h * HD + sub * E), w);
                    } else {
#pragma unroll
                        for (int e = 0; e < E; ++e) w[e] = 1.f;
                    }
                } else {
                    float ss = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
#pragma unroll
                    for (int off = LPH / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
                    r = rsqrtf(ss * (1.f / HD) + eps);
#pragma unroll
                    for (int e = 0; e < E; ++e) w[e] = is_q ? fwq[e] : fwk[e];
                }
                float a[E], o[E];
#pragma unroll
                for (int e = 0; e < E; ++e) a[e] = f[e] * r * w[e];
                if (HALF) {
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const float b = __shfl_sync(0xffffffffu, a[e], partner);
                        o[e] = a[e] * cs[e] + sgn * b * sn[e];
                    }
                } else {
#pragma unroll
                    for (int m = 0; m < P; ++m) {
                        o[2 * m] = a[2 * m] * cs[m] - a[2 * m + 1] * sn[m];
                        o[2 * m + 1] = a[2 * m] * sn[m] + a[2 * m + 1] * cs[m];
                    }
                }
                if (is_q)
                    st_stream(qo + (int64_t)vi * os.head + sub * E, pack<T>(o));
                else if (vi < n_vec)
                    st_stream(ko + (int64_t)(vi - n_heads) * os.head + sub * E, pack<T>(o));
            }
        }
    }
}

namespace {

constexpr int kExThreads = 256;

template <typename T, int LPH, bool ACROSS, bool HALF>
cudaError_t run_ex(void* q_out, void* k_out, const QkOutStrides& os, const void* q, const void* k,
                   int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                   int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                   int32_t n_heads, float eps, cudaStream_t s)
{
    constexpr int UNR = 8;
    const void* kfn = (const void*)k_qk_ex<T, LPH, UNR, ACROSS, HALF>;
    int64_t grid = (int64_t)ctas_per_sm(kfn, kExThreads, 0) * sm_count();
    const int64_t max_grid = (n_tokens + (kExThreads / 32) - 1) / (kExThreads / 32);
    if (grid > max_grid) grid = max_grid;
    if (grid < 1) grid = 1;
    k_qk_ex<T, LPH, UNR, ACROSS, HALF><<<(unsigned)grid, kExThreads, 0, s>>>(
        (T*)q_out, (T*)k_out, os, (const T*)q, (const T*)k, ld_q, ld_k, (const T*)wq, (const T*)wk, pos,
        grid_H, grid_W, tps, rope, n_tokens, n_heads, eps);
    return cudaGetLastError();
}

template <typename T, int LPH>
cudaError_t dispatch_opts(bool across, bool half, void* q_out, void* k_out, const QkOutStrides& os,
                          const void* q, const void* k, int64_t ld_q, int64_t ld_k, const void* wq,
                          const void* wk, const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps,
                          const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s)
{
#define ARGS q_out, k_out, os, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, n_tokens, n_heads, eps, s
    if (across) return half ? run_ex<T, LPH, true, true>(ARGS) : run_ex<T, LPH, true, false>(ARGS);
    return half ? run_ex<T, LPH, false, true>(ARGS) : run_ex<T, LPH, false, false>(ARGS);
#undef ARGS
}

}  // namespace

cudaError_t launch_qk_ex(sol_dtype dt, bool across, bool half, void* q_out, void* k_out,
                         const QkOutStrides& os, const void* q, const void* k, int64_t ld_q, int64_t ld_k,
                         const void* wq, const void* wk, const int32_t* pos, int32_t grid_H, int32_t grid_W,
                         int64_t tps, const RopeDev& rope, int64_t n_tokens, int32_t n_heads,
                         int32_t head_dim, float eps, cudaStream_t s)
{
    if (qk_cta_ex_fits(dt, half, n_heads, head_dim, q, k, n_tokens, tps, rope))  // staged rows (k_qk_cta.cu)
        return launch_qk_cta_ex(across, half, q_out, k_out, os, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps,
                                rope, n_tokens, n_heads, eps, s);
    const int lph = head_dim / (dt == SOL_DTYPE_BF16 ? 8 : 4);
#define ARGS across, half, q_out, k_out, os, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, n_tokens, n_heads, eps, s
    if (dt == SOL_DTYPE_BF16) {
        switch (lph) {
        case 8: return dispatch_opts<bf16, 8>(ARGS);
        case 16: return dispatch_opts<bf16, 16>(ARGS);
        case 32: return dispatch_opts<bf16, 32>(ARGS);
        default: return cudaErrorInvalidConfiguration;
        }
    }
    switch (lph) {
    case 8: return dispatch_opts<float, 8>(ARGS);
    case 16: return dispatch_opts<float, 16>(ARGS);
    case 32: return dispatch_opts<float, 32>(ARGS);
    default: return cudaErrorInvalidConfiguration;
    }
#undef ARGS
}

}  // namespace sol
