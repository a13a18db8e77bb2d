// k_rows.cu -- AdaLN modulation and the fused block prologue (gated residual -> AdaLN).
//
// One CTA per token row, rows walked with a grid stride.  The whole row lives in fp32
// registers (blockDim.x * U 16-byte vectors cover it), so x (and y) are read from HBM
// exactly once: the mean and then the variance are two reductions over registers
// (two-pass, so +-50 outliers and large offsets do not cancel), each a warp shuffle tree
// plus one shared-memory exchange.  The residual sum x' = x + gate*y stays unrounded in
// registers for the norm; only its stored copy is rounded.  Modulation rows come
// through the read-only path and stay L1/L2 resident across rows of the same sample.
#include "common.cuh"
#include "launch.h"

namespace sol {

template <typename T, int U, bool RESID>
__global__ void __launch_bounds__(512)
k_adaln_rows(T* x_out, int64_t ld_xo, T* h, int64_t ld_h, const T* x, int64_t ld_x,
             const T* __restrict__ y, int64_t ld_y, const T* __restrict__ gate,
             const T* __restrict__ shift, const T* __restrict__ scale, int64_t ld_mod, ModSel sel,
             int64_t n_tokens, int32_t vpr, float d, float eps)
{
    constexpr int E = Vec<T>::N;
    __shared__ float red[2][32];
    for (int64_t row = blockIdx.x; row < n_tokens; row += gridDim.x) {
        const int64_t mr = mod_row(row, sel);
        uint4 xr[U];
        uint4 yr[RESID ? U : 1];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = threadIdx.x + k * blockDim.x;
            if (col < vpr) {
                xr[k] = ld_stream(x + row * ld_x + (int64_t)col * E);
                if constexpr (RESID) yr[k] = ld_stream(y + row * ld_y + (int64_t)col * E);
            }
        }
        float v[U][E];
        float s = 0.f;
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = threadIdx.x + k * blockDim.x;
            if (col < vpr) {
                unpack<T>(xr[k], v[k]);
                if constexpr (RESID) {
                    float fy[E], fg[E];
                    unpack<T>(yr[k], fy);
                    if (gate) {
                        unpack<T>(ld_cached(gate + mr * ld_mod + (int64_t)col * E), fg);
                    } else {
#pragma unroll
                        for (int e = 0; e < E; ++e) fg[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < E; ++e) v[k][e] = fmaf(fg[e], fy[e], v[k][e]);
                    st_stream(x_out + row * ld_xo + (int64_t)col * E, pack<T>(v[k]));
                }
#pragma unroll
                for (int e = 0; e < E; ++e) s += v[k][e];
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) v[k][e] = 0.f;
            }
        }
        const float mean = block_sum(s, red[0]) / d;
        float q = 0.f;
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = threadIdx.x + k * blockDim.x;
            if (col < vpr) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float c = v[k][e] - mean;
                    q = fmaf(c, c, q);
                }
            }
        }
        const float var = block_sum(q, red[1]) / d;
        const float rstd = rsqrtf(var + eps);
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = threadIdx.x + k * blockDim.x;
            if (col < vpr) {
                float sh[E], sc[E];
                if (shift) {
                    unpack<T>(ld_cached(shift + mr * ld_mod + (int64_t)col * E), sh);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) sh[e] = 0.f;
                }
                if (scale) {
                    unpack<T>(ld_cached(scale + mr * ld_mod + (int64_t)col * E), sc);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) sc[e] = 0.f;
                }
                float o[E];
#pragma unroll
                for (int e = 0; e < E; ++e) o[e] = fmaf((v[k][e] - mean) * rstd, 1.f + sc[e], sh[e]);
                st_stream(h + row * ld_h + (int64_t)col * E, pack<T>(o));
            }
        }
    }
}

namespace {

constexpr int kMaxRowThreads = 512;
constexpr int kMaxRowU = 8;

struct RowShape {
    int threads, U;
};

// blockDim.x * U >= vpr with the fewest idle lanes; U preference 4, 5, 3, 2, 6, 8, 1, 7
// (enough independent loads per thread without crowding registers).
RowShape choose_row_shape(int64_t vpr)
{
    static const int kU[] = {4, 5, 3, 2, 6, 8, 1, 7};
    RowShape best{0, 0};
    int64_t best_waste = -1;
    for (int ui = 0; ui < 8; ++ui) {
        const int U = kU[ui];
        int64_t t = (vpr + U - 1) / U;
        t = (t + 31) / 32 * 32;
        if (t > kMaxRowThreads) continue;
        const int64_t waste = t * U - vpr;
        if (best_waste < 0 || waste < best_waste) {
            best = RowShape{(int)t, U};
            best_waste = waste;
        }
    }
    return best;
}

template <typename T, int U, bool RESID>
cudaError_t run_rows(void* x_out, int64_t ld_xo, void* h, int64_t ld_h, const void* x,
                     int64_t ld_x, const void* y, int64_t ld_y, const void* gate,
                     const void* shift, const void* scale, int64_t ld_mod, const ModSel& sel,
                     int64_t n_tokens, int64_t vpr, int threads, int64_t d, float eps,
                     cudaStream_t s)
{
    const void* kfn = (const void*)k_adaln_rows<T, U, RESID>;
    int64_t grid = (int64_t)ctas_per_sm(kfn, threads, 0) * sm_count();
    if (grid < 1) grid = 1;
    if (grid > n_tokens) grid = n_tokens;
    k_adaln_rows<T, U, RESID><<<(unsigned)grid, threads, 0, s>>>(
        (T*)x_out, ld_xo, (T*)h, ld_h, (const T*)x, ld_x, (const T*)y, ld_y, (const T*)gate,
        (const T*)shift, (const T*)scale, ld_mod, sel, n_tokens, (int32_t)vpr, (float)d, eps);
    return cudaGetLastError();
}

template <typename T, bool RESID>
cudaError_t dispatch_u(const RowShape& sh, void* x_out, int64_t ld_xo, void* h, int64_t ld_h,
                       const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                       const void* gate, const void* shift, const void* scale, int64_t ld_mod,
                       const ModSel& sel, int64_t n_tokens, int64_t vpr, int64_t d, float eps,
                       cudaStream_t s)
{
#define CASE(U)                                                                                  \
    case U:                                                                                      \
        return run_rows<T, U, RESID>(x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift,      \
                                     scale, ld_mod, sel, n_tokens, vpr, sh.threads, d, eps, s);
    switch (sh.U) {
        CASE(1) CASE(2) CASE(3) CASE(4) CASE(5) CASE(6) CASE(7) CASE(8)
    default: return cudaErrorInvalidConfiguration;
    }
#undef CASE
}

}  // namespace

bool adaln_row_fits(int64_t vpr) { return vpr >= 1 && vpr <= (int64_t)kMaxRowThreads * kMaxRowU; }

cudaError_t launch_adaln_rows(sol_dtype dt, void* x_out, int64_t ld_xo, void* h, int64_t ld_h,
                              const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                              const void* gate, const void* shift, const void* scale,
                              int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                              float eps, cudaStream_t s)
{
    const int64_t vpr = d / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const RowShape sh = choose_row_shape(vpr);
    if (sh.threads == 0) return cudaErrorInvalidConfiguration;
    if (dt == SOL_DTYPE_BF16) {
        if (y)
            return dispatch_u<bf16, true>(sh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift,
                                          scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
        return dispatch_u<bf16, false>(sh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift,
                                       scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
    }
    if (y)
        return dispatch_u<float, true>(sh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift,
                                       scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
    return dispatch_u<float, false>(sh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift,
                                    scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
}

}  // namespace sol
