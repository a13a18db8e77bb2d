// k_stream.cu -- streaming per-token kernels: the gated residual and the SwiGLU
// activation.  Both are pure HBM streams (2 reads : 1 write per element), so the design
// is about bytes in flight and coalescing, not arithmetic:
//   * every access is a 16-byte vector; consecutive threads touch consecutive vectors;
//   * a CTA owns one fixed column chunk (blockDim.x * U vectors) of a row and never
//     changes columns.  The gated residual and SwiGLU launch one CTA per (row, chunk), so
//     the hardware refills each SM as CTAs retire; at 245,952 tokens this streams 16-22%
//     faster on B200 than a persistent grid walking rows with a stride (SwiGLU 5.8 -> 7.1
//     TB/s, gated residual 6.1 -> 7.05 TB/s).  The Cache-DiT variant gives each CTA a
//     contiguous run of 8 rows, so that its per-sample fp64 sums cost one atomic per warp
//     and sum per run rather than per row;
//   * each thread issues all U x inputs loads before the first use (U * 32 bytes in
//     flight per thread); inputs nothing in the kernel writes come through the
//     read-only path, outputs are stored without L1 allocation;
//   * the gate row is re-read through the read-only path and stays L1/L2 resident.
#include "common.cuh"
#include "launch.h"

// First choice of 16-byte vectors per thread and input (U), per kernel, from a sweep on
// B200 at 245,952 tokens: the gated residual (d 5120) streams 7.17-7.18 TB/s with U = 2
// against 7.05-7.06 with U = 4 or 8; SwiGLU (d 13,824) 7.13-7.14 with U = 4..8 against
// 6.45-6.48 with U = 2.
#ifndef SOL_GATED_UPREF_FIRST
#define SOL_GATED_UPREF_FIRST 2
#endif
// Rows per CTA of the Cache-DiT variant, from a sweep on B200 (245,952 x 5120, refresh):
// 8: 1.92 ms; 32: 1.98; a persistent-sized run (0): 2.11; 2: 3.80 (the per-warp fp64
// atomics then contend).
#ifndef SOL_DIFF_ROWS_PER_CTA
#define SOL_DIFF_ROWS_PER_CTA 8
#endif
#ifndef SOL_STREAM_UPREF_FIRST
#define SOL_STREAM_UPREF_FIRST 4  // SwiGLU and the Cache-DiT variant
#endif

namespace sol {

// Gated residual [XHH-QA "门控残差"]: out = x + gate[r] * y, fp32 inside.  RO: out does
// not alias x, so x may come through the read-only path (y never aliases out).
template <typename T, int U, bool RO>
__global__ void __launch_bounds__(512)
k_gated_residual(T* __restrict__ out, int64_t ld_out, const T* x, int64_t ld_x,
                 const T* __restrict__ y, int64_t ld_y, const T* __restrict__ gate,
                 int64_t ld_mod, ModSel sel, int64_t n_tokens, int32_t vpr, int32_t cpr)
{
    constexpr int E = Vec<T>::N;
    const int chunk = blockIdx.x % cpr;
    const int64_t row_step = gridDim.x / cpr;
    const int col0 = chunk * blockDim.x * U + threadIdx.x;
    for (int64_t row = blockIdx.x / cpr; row < n_tokens; row += row_step) {
        const int64_t mr = mod_row(row, sel);
        uint4 xv[U], yv[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                xv[k] = RO ? ld_stream_ro(x + row * ld_x + (int64_t)col * E)
                           : ld_stream(x + row * ld_x + (int64_t)col * E);
                yv[k] = ld_stream_ro(y + row * ld_y + (int64_t)col * E);
            }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                float fx[E], fy[E], fg[E];
                unpack<T>(xv[k], fx);
                unpack<T>(yv[k], fy);
                if (gate) {
                    unpack<T>(ld_cached(gate + mr * ld_mod + (int64_t)col * E), fg);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) fg[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < E; ++e) fx[e] = fmaf(fg[e], fy[e], fx[e]);
                st_stream(out + row * ld_out + (int64_t)col * E, pack<T>(fx));
            }
        }
    }
}

// Gated residual fused with the Cache-DiT residual-change statistics: out = x + gate*y as
// in k_gated_residual; r = gate*y is compared with the cached residual of the previous
// step, sums[s] += (sum |r - cache|, sum |cache|) over sample s, and with REFRESH the
// cache is overwritten by r.  Each thread keeps fp32 partials per row and folds them into
// fp64 accumulators; a CTA walks a contiguous run of rows_per_cta rows, and when it moves
// to another sample (and at the end) every warp adds its fp64 totals with one atomicAdd
// per sum, so no block barrier is needed.
template <typename T, int U, bool REFRESH>
__global__ void __launch_bounds__(512)
k_gated_residual_diff(T* __restrict__ out, int64_t ld_out, const T* x, int64_t ld_x,
                      const T* __restrict__ y, int64_t ld_y, const T* __restrict__ gate,
                      int64_t ld_mod, T* cache, int64_t ld_c, double* __restrict__ sums,
                      ModSel sel, int64_t n_tokens, int32_t vpr, int32_t cpr, int64_t rows_per_cta)
{
    constexpr int E = Vec<T>::N;
    const int chunk = blockIdx.x % cpr;
    const int col0 = chunk * blockDim.x * U + threadIdx.x;
    const int64_t row0 = (int64_t)(blockIdx.x / cpr) * rows_per_cta;
    const int64_t row1 = row0 + rows_per_cta < n_tokens ? row0 + rows_per_cta : n_tokens;
    double acc_d = 0.0, acc_c = 0.0;
    int64_t cur = -1;
    auto flush = [&]() {
        double td = acc_d, tc = acc_c;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            td += __shfl_xor_sync(0xffffffffu, td, off);
            tc += __shfl_xor_sync(0xffffffffu, tc, off);
        }
        if ((threadIdx.x & 31) == 0 && cur >= 0) {
            atomicAdd(sums + 2 * cur, td);
            atomicAdd(sums + 2 * cur + 1, tc);
        }
        acc_d = 0.0;
        acc_c = 0.0;
    };
    for (int64_t row = row0; row < row1; ++row) {  // a contiguous run of rows per CTA
        const int64_t mr = mod_row(row, sel);
        const int64_t sample = sample_of(row, sel);
        if (sample != cur) {  // uniform across the CTA
            flush();
            cur = sample;
        }
        uint4 xv[U], yv[U], cv[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                xv[k] = ld_stream(x + row * ld_x + (int64_t)col * E);
                yv[k] = ld_stream_ro(y + row * ld_y + (int64_t)col * E);
                cv[k] = ld_stream(cache + row * ld_c + (int64_t)col * E);
            }
        }
        float pd = 0.f, pc = 0.f;
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                float fx[E], fy[E], fg[E], fc[E], fr[E];
                unpack<T>(xv[k], fx);
                unpack<T>(yv[k], fy);
                unpack<T>(cv[k], fc);
                if (gate) {
                    unpack<T>(ld_cached(gate + mr * ld_mod + (int64_t)col * E), fg);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) fg[e] = 0.f;
                }
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    fr[e] = fg[e] * fy[e];
                    fx[e] = fmaf(fg[e], fy[e], fx[e]);
                    pd += fabsf(fr[e] - fc[e]);
                    pc += fabsf(fc[e]);
                }
                st_stream(out + row * ld_out + (int64_t)col * E, pack<T>(fx));
                if constexpr (REFRESH) st_stream(cache + row * ld_c + (int64_t)col * E, pack<T>(fr));
            }
        }
        acc_d += (double)pd;
        acc_c += (double)pc;
    }
    flush();
}

// The two MUFU operations of the bf16 SwiGLU: 2^x and 1/x, approximate (relative
// error ~2^-22), flushing subnormal results to zero.  1/inf = 0, so a very negative
// pre-activation gives silu = -0 as its limit.
__device__ __forceinline__ float exp2f_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// silu(a) * b.  bf16 outputs: ex2.approx-based exponential and approximate division
// (one MUFU op each); the relative error is a few 1e-7, far below a bf16 ulp.  f32
// outputs: expf and IEEE division.
template <typename T> __device__ __forceinline__ float silu_mul(float a, float b);
template <> __device__ __forceinline__ float silu_mul<bf16>(float a, float b)
{
    return __fdividef(a, 1.f + __expf(-a)) * b;
}
template <> __device__ __forceinline__ float silu_mul<float>(float a, float b)
{
    return a / (1.f + expf(-a)) * b;
}

// SwiGLU [XHH-QA, STM-GAN]: out_j = silu(a_j) * b_j.  MAXT / MINB: launch bounds; blocks of
// at most 288 threads are compiled for three resident CTAs per SM (72 registers instead of
// 76, which allow two), keeping a third row in flight (bf16 d 13,824, 245,952 tokens:
// +2.3% under the persistent grid this kernel used to run on).
template <typename T, int U, int MAXT, int MINB>
__global__ void __launch_bounds__(MAXT, MINB)
k_swiglu(T* __restrict__ out, int64_t ld_out, const T* __restrict__ a, const T* __restrict__ b,
         int64_t ld_in, int64_t n_tokens, int32_t vpr, int32_t cpr)
{
    constexpr int E = Vec<T>::N;
    const int chunk = blockIdx.x % cpr;
    const int64_t row_step = gridDim.x / cpr;
    const int col0 = chunk * blockDim.x * U + threadIdx.x;
    for (int64_t row = blockIdx.x / cpr; row < n_tokens; row += row_step) {
        uint4 av[U], bv[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                av[k] = ld_stream_ro(a + row * ld_in + (int64_t)col * E);
                bv[k] = ld_stream_ro(b + row * ld_in + (int64_t)col * E);
            }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const int col = col0 + k * blockDim.x;
            if (col < vpr) {
                if constexpr (sizeof(T) == 2) {
                    // a * b / (1 + 2^(-a*log2 e)): products and the sum in packed f32x2,
                    // exp2 and the reciprocal on the MUFU pipe
                    float2 fa[E / 2], fb[E / 2];
                    unpack2<T>(av[k], fa);
                    unpack2<T>(bv[k], fb);
                    const float2 nl2e = make_float2(-1.4426950408889634f, -1.4426950408889634f);
#pragma unroll
                    for (int i = 0; i < E / 2; ++i) {
                        const float2 t = __fmul2_rn(fa[i], nl2e);
                        const float2 den = __fadd2_rn(make_float2(exp2f_approx(t.x), exp2f_approx(t.y)),
                                                      make_float2(1.f, 1.f));
                        const float2 ab = __fmul2_rn(fa[i], fb[i]);
                        fa[i] = __fmul2_rn(ab, make_float2(rcp_approx(den.x), rcp_approx(den.y)));
                    }
                    st_stream(out + row * ld_out + (int64_t)col * E, pack2<T>(fa));
                } else {
                    float fa[E], fb[E];
                    unpack<T>(av[k], fa);
                    unpack<T>(bv[k], fb);
#pragma unroll
                    for (int e = 0; e < E; ++e) fa[e] = silu_mul<T>(fa[e], fb[e]);
                    st_stream(out + row * ld_out + (int64_t)col * E, pack<T>(fa));
                }
            }
        }
    }
}

namespace {

struct StreamShape {
    int threads, U, cpr;
};

// Column chunking of a row of `vpr` vectors: the fewest idle lanes, then U in the
// preference order below (first_u moved to the front), then blockDim nearest 256.
StreamShape choose_stream_shape(int64_t vpr, int first_u)
{
    int kU[] = {4, 6, 8, 3, 2, 1};
    for (int i = 0; i < 6; ++i)
        if (kU[i] == first_u) {
            for (int j = i; j > 0; --j) kU[j] = kU[j - 1];
            kU[0] = first_u;
        }
    StreamShape best{0, 0, 0};
    int64_t best_waste = -1;
    int best_rank = 0, best_tdist = 0;
    for (int ui = 0; ui < 6; ++ui) {
        for (int t = 32; t <= 512; t += 32) {
            const int64_t chunk = (int64_t)t * kU[ui];
            const int64_t cpr = (vpr + chunk - 1) / chunk;
            const int64_t waste = cpr * chunk - vpr;
            const int tdist = t > 256 ? t - 256 : 256 - t;
            const bool better = best_waste < 0 || waste < best_waste ||
                                (waste == best_waste &&
                                 (ui < best_rank || (ui == best_rank && tdist < best_tdist)));
            if (better) {
                best = StreamShape{t, kU[ui], (int)cpr};
                best_waste = waste;
                best_rank = ui;
                best_tdist = tdist;
            }
        }
    }
    return best;
}

// One CTA per row chunk (capped at the grid limit; the kernels' row loop covers the rest).
// The hardware then refills each SM as its CTAs retire, which streams measurably faster on
// B200 than a persistent grid whose CTAs walk rows with a stride.
int64_t flat_grid(const StreamShape& sh, int64_t n_tokens)
{
    const int64_t max_rows = 0x7fffffffLL / sh.cpr;
    return (n_tokens < max_rows ? n_tokens : max_rows) * sh.cpr;
}

int64_t stream_grid(const void* kernel, const StreamShape& sh, int64_t n_tokens)
{
    const int64_t resident = (int64_t)ctas_per_sm(kernel, sh.threads, 0) * sm_count();
    int64_t rows = resident / sh.cpr;
    if (rows < 1) rows = 1;
    if (rows > n_tokens) rows = n_tokens;
    return rows * sh.cpr;
}

template <typename T, int U, bool RO>
cudaError_t run_gated_ro(void* out, int64_t ld_out, const void* x, int64_t ld_x, const void* y,
                         int64_t ld_y, const void* gate, int64_t ld_mod, const ModSel& sel,
                         int64_t n_tokens, int64_t vpr, const StreamShape& sh, cudaStream_t s)
{
    const int64_t grid = flat_grid(sh, n_tokens);
    k_gated_residual<T, U, RO><<<(unsigned)grid, sh.threads, 0, s>>>(
        (T*)out, ld_out, (const T*)x, ld_x, (const T*)y, ld_y, (const T*)gate, ld_mod, sel,
        n_tokens, (int32_t)vpr, sh.cpr);
    return cudaGetLastError();
}

template <typename T, int U>
cudaError_t run_gated(void* out, int64_t ld_out, const void* x, int64_t ld_x, const void* y,
                      int64_t ld_y, const void* gate, int64_t ld_mod, const ModSel& sel,
                      int64_t n_tokens, int64_t vpr, const StreamShape& sh, cudaStream_t s)
{
    if (out == x)
        return run_gated_ro<T, U, false>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, sel, n_tokens,
                                         vpr, sh, s);
    return run_gated_ro<T, U, true>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, sel, n_tokens, vpr,
                                    sh, s);
}

template <typename T, int U, int MAXT, int MINB>
cudaError_t run_swiglu_bounds(void* out, int64_t ld_out, const void* a, const void* b, int64_t ld_in,
                              int64_t n_tokens, int64_t vpr, const StreamShape& sh, cudaStream_t s)
{
    const int64_t grid = flat_grid(sh, n_tokens);
    k_swiglu<T, U, MAXT, MINB><<<(unsigned)grid, sh.threads, 0, s>>>((T*)out, ld_out, (const T*)a,
                                                                      (const T*)b, ld_in, n_tokens,
                                                                      (int32_t)vpr, sh.cpr);
    return cudaGetLastError();
}

template <typename T, int U>
cudaError_t run_swiglu(void* out, int64_t ld_out, const void* a, const void* b, int64_t ld_in,
                       int64_t n_tokens, int64_t vpr, const StreamShape& sh, cudaStream_t s)
{
    if (sh.threads <= 288)
        return run_swiglu_bounds<T, U, 288, 3>(out, ld_out, a, b, ld_in, n_tokens, vpr, sh, s);
    return run_swiglu_bounds<T, U, 512, 1>(out, ld_out, a, b, ld_in, n_tokens, vpr, sh, s);
}

#define SOL_DISPATCH_U(U_, CALL) \
    switch (U_) {                \
    case 1: return CALL(1);      \
    case 2: return CALL(2);      \
    case 3: return CALL(3);      \
    case 4: return CALL(4);      \
    case 6: return CALL(6);      \
    case 8: return CALL(8);      \
    default: return cudaErrorInvalidConfiguration; \
    }

}  // namespace

cudaError_t launch_gated_residual(sol_dtype dt, void* out, int64_t ld_out, const void* x,
                                  int64_t ld_x, const void* y, int64_t ld_y, const void* gate,
                                  int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                                  cudaStream_t s)
{
    const int64_t vpr = d / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const StreamShape sh = choose_stream_shape(vpr, SOL_GATED_UPREF_FIRST);
#define CALL_B(U) run_gated<bf16, U>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, sel, n_tokens, vpr, sh, s)
#define CALL_F(U) run_gated<float, U>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, sel, n_tokens, vpr, sh, s)
    if (dt == SOL_DTYPE_BF16) {
        SOL_DISPATCH_U(sh.U, CALL_B)
    }
    SOL_DISPATCH_U(sh.U, CALL_F)
#undef CALL_B
#undef CALL_F
}

namespace {
template <typename T, int U, bool REFRESH>
cudaError_t run_diff(void* out, int64_t ld_out, const void* x, int64_t ld_x, const void* y,
                     int64_t ld_y, const void* gate, int64_t ld_mod, void* cache, int64_t ld_c,
                     double* sums, const ModSel& sel, int64_t n_tokens, int64_t vpr,
                     const StreamShape& sh, cudaStream_t s)
{
    if (n_tokens <= 0) return cudaSuccess;
    // Rows per CTA: SOL_DIFF_ROWS_PER_CTA, or (0) as many as a grid of resident CTAs needs.
    int64_t rows = SOL_DIFF_ROWS_PER_CTA;
    if (rows <= 0) {
        const void* kfn = (const void*)k_gated_residual_diff<T, U, REFRESH>;
        const int64_t groups = stream_grid(kfn, sh, n_tokens) / sh.cpr;
        rows = (n_tokens + groups - 1) / groups;
    }
    const int64_t max_groups = 0x7fffffffLL / sh.cpr;
    if ((n_tokens + rows - 1) / rows > max_groups) rows = (n_tokens + max_groups - 1) / max_groups;
    const int64_t grid = (n_tokens + rows - 1) / rows * sh.cpr;
    k_gated_residual_diff<T, U, REFRESH><<<(unsigned)grid, sh.threads, 0, s>>>(
        (T*)out, ld_out, (const T*)x, ld_x, (const T*)y, ld_y, (const T*)gate, ld_mod, (T*)cache, ld_c,
        sums, sel, n_tokens, (int32_t)vpr, sh.cpr, rows);
    return cudaGetLastError();
}

template <typename T, int U>
cudaError_t run_diff_r(bool refresh, void* out, int64_t ld_out, const void* x, int64_t ld_x,
                       const void* y, int64_t ld_y, const void* gate, int64_t ld_mod, void* cache,
                       int64_t ld_c, double* sums, const ModSel& sel, int64_t n_tokens, int64_t vpr,
                       const StreamShape& sh, cudaStream_t s)
{
    if (refresh)
        return run_diff<T, U, true>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, cache, ld_c, sums, sel,
                                    n_tokens, vpr, sh, s);
    return run_diff<T, U, false>(out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, cache, ld_c, sums, sel,
                                 n_tokens, vpr, sh, s);
}
}  // namespace

cudaError_t launch_gated_residual_diff(sol_dtype dt, void* out, int64_t ld_out, const void* x,
                                       int64_t ld_x, const void* y, int64_t ld_y, const void* gate,
                                       int64_t ld_mod, void* cache, int64_t ld_c, bool refresh,
                                       double* sums, const ModSel& sel, int64_t n_tokens, int64_t d,
                                       cudaStream_t s)
{
    const int64_t vpr = d / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const StreamShape sh = choose_stream_shape(vpr, SOL_STREAM_UPREF_FIRST);
#define CALL_B(U) run_diff_r<bf16, U>(refresh, out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, cache, ld_c, sums, sel, n_tokens, vpr, sh, s)
#define CALL_F(U) run_diff_r<float, U>(refresh, out, ld_out, x, ld_x, y, ld_y, gate, ld_mod, cache, ld_c, sums, sel, n_tokens, vpr, sh, s)
    if (dt == SOL_DTYPE_BF16) {
        SOL_DISPATCH_U(sh.U, CALL_B)
    }
    SOL_DISPATCH_U(sh.U, CALL_F)
#undef CALL_B
#undef CALL_F
}

cudaError_t launch_swiglu(sol_dtype dt, void* out, int64_t ld_out, const void* a, const void* b,
                          int64_t ld_in, int64_t n_tokens, int64_t inner, cudaStream_t s)
{
    const int64_t vpr = inner / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const StreamShape sh = choose_stream_shape(vpr, SOL_STREAM_UPREF_FIRST);
#define CALL_B(U) run_swiglu<bf16, U>(out, ld_out, a, b, ld_in, n_tokens, vpr, sh, s)
#define CALL_F(U) run_swiglu<float, U>(out, ld_out, a, b, ld_in, n_tokens, vpr, sh, s)
    if (dt == SOL_DTYPE_BF16) {
        SOL_DISPATCH_U(sh.U, CALL_B)
    }
    SOL_DISPATCH_U(sh.U, CALL_F)
#undef CALL_B
#undef CALL_F
}

}  // namespace sol
