// k_adaln_warp.cu -- AdaLN modulation (bf16) with one warp per token row, the whole row
// held in registers.
//
// [XHH-QA] "8xH200 上的 MiniMax-H3" (xhh.club), Q&A on the fused kernels: AdaLN
// modulation.  Per row: mean, biased variance by a second pass over the registers (no
// cancellation from outliers), then h = (x - mean) * rstd * (1 + scale[r]) + shift[r].
//
// Lane l holds 16-byte vectors l, l + 32, ..., so every warp-wide load and store covers
// 512 contiguous bytes; the reductions are warp shuffles only (no shared memory, no
// barrier).  With VPL vectors per lane a row is 256 * VPL elements (d = 5120: VPL = 20,
// 80 registers of packed bf16).  Arithmetic is f32x2; the row is widened from its
// packed form in each of the three passes instead of being kept in fp32 (which would
// double the registers and halve the rows in flight).  h may be x itself: a row is read
// completely before any of it is written.  Used for bf16 AdaLN with d a multiple of 256
// (up to 6144) that the four-warp kernel below does not take; the bulk-copy ring kernel
// (k_rows.cu) takes fp32, other widths and the prologues that are not register-resident.
//
// The four-warp kernel (k_prologue_regs) serves the fused prologue and, without its
// residual, plain AdaLN too (d a multiple of 1024 up to 6144, h and x with one row
// stride): a quarter row per warp fits in fp32 registers, so x is widened once instead of
// in each of three passes, and 64 registers allow 8 CTAs (32 warps) per SM.  At 245,952 x
// 5120: 0.740 ms (6.81 TB/s) alone against 0.777 for the one-warp kernel, and 0.815 vs
// 0.854 ms inside 100 back-to-back block passes under the power cap.
//
// Both kernels here launch one CTA per row (or per block of rows) instead of a persistent
// grid: SMs are refilled as CTAs retire, which at 245,952 x 5120 measured AdaLN 6.30 ->
// 6.43 TB/s and the prologue 6.33 -> 6.73 TB/s on B200 (the launch shapes below were
// swept under the persistent grid).
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"

// Launch shape, from sweeps on B200 at 245,952 x 5120 tokens (alone, full clock).  With
// one CTA per row block: one warp per CTA, >= 8 per SM: 6.56 TB/s; 64 x 4: 6.49-6.50;
// 128 x 2: 6.42.  (Under the earlier persistent grid: 64 x 4: 6.39-6.48; 256 x 1:
// 6.25-6.46; 128 x 3, capped at 168 registers and spilling: 5.99-6.13.)  The row needs
// ~226 registers per lane unspilled.
#ifndef SOL_ADALN_WARP_BLOCK
#define SOL_ADALN_WARP_BLOCK 32
#endif
#ifndef SOL_ADALN_WARP_MINB
#define SOL_ADALN_WARP_MINB 8
#endif
// Fused prologue, from the same sweeps (x, y at 245,952 x 5120): 4 warps per row, one CTA
// per row, x' kept in fp32 registers, >= 6 CTAs per SM (80 registers): 1.48 ms alone, 1.50
// ms inside 100 back-to-back block passes under the power cap (~1.6 GHz).  The same with 5
// CTAs per SM: 1.48 / 1.52; with 4 (120 registers): 1.80 under the cap.  x' re-formed
// from the packed inputs in every pass (126 registers, 4 per SM): 1.49-1.50 / 1.57.
// Earlier, persistent grid: 6.40-6.54 TB/s; 2 warps per row (222 registers): 6.06-6.10;
// the ring kernel: 5.92-6.31.
#ifndef SOL_PROLOGUE_REGS_MINB
#define SOL_PROLOGUE_REGS_MINB 6
#endif
#ifndef SOL_ADALN4_MINB
#define SOL_ADALN4_MINB 8  // the same kernel without the residual (plain AdaLN); 10 or 12 spill: 3.0-3.7 TB/s
#endif
#ifndef SOL_PROLOGUE_REGS_WPR
#define SOL_PROLOGUE_REGS_WPR 4  // warps per row of the fused prologue
#endif

namespace sol {

template <int VPL>
__global__ void __launch_bounds__(SOL_ADALN_WARP_BLOCK, SOL_ADALN_WARP_MINB) k_adaln_warp(bf16* h, int64_t ld_h, const bf16* x, int64_t ld_x,
                                                    const bf16* shift, const bf16* scale, int64_t ld_mod,
                                                    ModSel sel, int64_t n_tokens, float eps)
{
    constexpr int D = 256 * VPL;
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t wstep = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row = w0; row < n_tokens; row += wstep) {
        // the modulation row first: with per-token stream ids its load is then in flight
        // with the row's, not on the critical path after the reductions
        const int64_t r = mod_row(row, sel);
        uint4 xv[VPL];
        const bf16* xr = x + row * ld_x + 8 * lane;
#pragma unroll
        for (int i = 0; i < VPL; ++i) xv[i] = ld_stream(xr + 256 * i);

        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            float2 f[4];
            unpack2<bf16>(xv[i], f);
#pragma unroll
            for (int e = 0; e < 4; ++e) s2 = __fadd2_rn(s2, f[e]);
        }
        const float mu = warp_sum(s2.x + s2.y) * (1.f / D);
        const float2 mu2 = make_float2(-mu, -mu);
        float2 q2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            float2 f[4];
            unpack2<bf16>(xv[i], f);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 c = __fadd2_rn(f[e], mu2);
                q2 = __ffma2_rn(c, c, q2);
            }
        }
        const float rs = rsqrtf(warp_sum(q2.x + q2.y) * (1.f / D) + eps);
        const float2 a2 = make_float2(rs, rs), c2 = make_float2(-mu * rs, -mu * rs);

        const bf16* sc = scale ? scale + r * ld_mod + 8 * lane : nullptr;
        const bf16* sh = shift ? shift + r * ld_mod + 8 * lane : nullptr;
        bf16* hr = h + row * ld_h + 8 * lane;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            float2 f[4], g[4], b[4], o[4];
            unpack2<bf16>(xv[i], f);
            if (sc) {
                unpack2<bf16>(ld_cached(sc + 256 * i), g);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) g[e] = make_float2(0.f, 0.f);
            }
            if (sh) {
                unpack2<bf16>(ld_cached(sh + 256 * i), b);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) b[e] = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[e] = __ffma2_rn(__ffma2_rn(f[e], a2, c2), __fadd2_rn(make_float2(1.f, 1.f), g[e]), b[e]);
            st_stream(hr + 256 * i, pack2<bf16>(o));
        }
    }
}

// Fused prologue x' = x + gate[r] * y, h = AdaLN(x') (bf16) with one CTA of WPR warps per
// row: each warp loads its 1/WPR of the row -- x, y and the gate row, VPH 16-byte vectors
// of each per lane (d = 256 * VPH * WPR) -- forms x' once in fp32 registers (d = 5120 with
// four warps: 40 registers; never rounded before the norm) and reads it in the two later
// passes.  x_out (x' rounded) is written in the first pass, h in the last; x_out may be x
// (a lane overwrites only elements it has already read).  The warps' sums meet in shared
// memory, one barrier per reduction.
// RES = false: plain AdaLN of x (no residual, no x_out) in the same four-warp form.
template <int VPH, int WPR, bool RES>
__global__ void __launch_bounds__(32 * WPR, RES ? SOL_PROLOGUE_REGS_MINB : SOL_ADALN4_MINB)
    k_prologue_regs(bf16* x_out, int64_t ld_xo, bf16* h, int64_t ld_h, const bf16* x, int64_t ld_x, const bf16* y,
                    int64_t ld_y, const bf16* gate, const bf16* shift, const bf16* scale, int64_t ld_mod,
                    ModSel sel, int64_t n_tokens, float eps)
{
    constexpr int D = 256 * VPH * WPR;
    __shared__ float red[2][WPR];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int col = warp * (256 * VPH) + 8 * lane;  // this lane's first element; vector i at + 256 i
    for (int64_t row = blockIdx.x; row < n_tokens; row += gridDim.x) {
        const int64_t r = mod_row(row, sel);
        uint4 xv[VPH], yv[VPH], gv[VPH];
        const bf16* xr = x + row * ld_x + col;
        const bf16* yr = y + row * ld_y + col;
#pragma unroll
        for (int i = 0; i < VPH; ++i) {
            xv[i] = ld_stream(xr + 256 * i);
            if (RES) yv[i] = ld_stream(yr + 256 * i);
        }
        const bf16* gr = RES && gate ? gate + r * ld_mod + col : nullptr;
#pragma unroll
        for (int i = 0; i < VPH; ++i) gv[i] = gr ? ld_cached(gr + 256 * i) : make_uint4(0u, 0u, 0u, 0u);

        // x' = x + gate * y once, kept in fp32 (never rounded before the norm); x_out gets
        // its rounding at once -- a lane overwrites only what it has already read
        bf16* xo = RES ? x_out + row * ld_xo + col : nullptr;  // no x_out without the residual
        float2 xp[VPH][4];
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VPH; ++i) {
            float2 fx[4];
            unpack2<bf16>(xv[i], fx);
            if constexpr (RES) {
                float2 fy[4], fg[4];
                unpack2<bf16>(yv[i], fy);
                unpack2<bf16>(gv[i], fg);
#pragma unroll
                for (int e = 0; e < 4; ++e) xp[i][e] = __ffma2_rn(fg[e], fy[e], fx[e]);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) xp[i][e] = fx[e];
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) s2 = __fadd2_rn(s2, xp[i][e]);
            if (RES) st_stream(xo + 256 * i, pack2<bf16>(xp[i]));
        }
        float t = warp_sum(s2.x + s2.y);
        if (lane == 0) red[0][warp] = t;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int k = 0; k < WPR; ++k) tot += red[0][k];
        const float mu = tot * (1.f / D);
        const float2 mu2 = make_float2(-mu, -mu);
        float2 q2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < VPH; ++i) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 c = __fadd2_rn(xp[i][e], mu2);
                q2 = __ffma2_rn(c, c, q2);
            }
        }
        t = warp_sum(q2.x + q2.y);
        if (lane == 0) red[1][warp] = t;
        __syncthreads();
        tot = 0.f;
#pragma unroll
        for (int k = 0; k < WPR; ++k) tot += red[1][k];
        const float rs = rsqrtf(tot * (1.f / D) + eps);
        const float2 a2 = make_float2(rs, rs), c2 = make_float2(-mu * rs, -mu * rs);
        const bf16* sc = scale ? scale + r * ld_mod + col : nullptr;
        const bf16* sh = shift ? shift + r * ld_mod + col : nullptr;
        bf16* hr = h + row * ld_h + col;
#pragma unroll
        for (int i = 0; i < VPH; ++i) {
            float2 m1[4], m0[4], o[4];
            if (sc) {
                unpack2<bf16>(ld_cached(sc + 256 * i), m1);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) m1[e] = make_float2(0.f, 0.f);
            }
            if (sh) {
                unpack2<bf16>(ld_cached(sh + 256 * i), m0);
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) m0[e] = make_float2(0.f, 0.f);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e)
                o[e] = __ffma2_rn(__ffma2_rn(xp[i][e], a2, c2), __fadd2_rn(make_float2(1.f, 1.f), m1[e]), m0[e]);
            st_stream(hr + 256 * i, pack2<bf16>(o));
        }
    }
}

namespace {

template <int VPL>
cudaError_t launch_vpl(void* h, int64_t ld_h, const void* x, int64_t ld_x, const void* shift, const void* scale,
                       int64_t ld_mod, const ModSel& sel, int64_t n_tokens, float eps, cudaStream_t s)
{
    auto kern = k_adaln_warp<VPL>;
    constexpr int block = SOL_ADALN_WARP_BLOCK;
    const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), block, 0);
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t rows_per_cta = block / 32;
    // one CTA per rows_per_cta rows (the row loop covers what the grid limit leaves): the
    // hardware refills SMs as CTAs retire, which streams faster than a persistent grid
    const int64_t grid = std::min<int64_t>(0x7fffffffLL, (n_tokens + rows_per_cta - 1) / rows_per_cta);
    kern<<<(unsigned)grid, block, 0, s>>>(static_cast<bf16*>(h), ld_h, static_cast<const bf16*>(x), ld_x,
                                        static_cast<const bf16*>(shift), static_cast<const bf16*>(scale), ld_mod,
                                        sel, n_tokens, eps);
    return cudaGetLastError();
}

template <int VPH, int WPR, bool RES>
cudaError_t launch_pro_vph(void* x_out, void* h, const void* x, const void* y, const void* gate, const void* shift,
                           const void* scale, int64_t ld, int64_t ld_mod, const ModSel& sel, int64_t n_tokens,
                           float eps, cudaStream_t s)
{
    auto kern = k_prologue_regs<VPH, WPR, RES>;
    const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), 32 * WPR, 0);
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t grid = std::min<int64_t>(0x7fffffffLL, n_tokens);  // one CTA per row, as above
    kern<<<(unsigned)grid, 32 * WPR, 0, s>>>(static_cast<bf16*>(x_out), ld, static_cast<bf16*>(h), ld,
                                       static_cast<const bf16*>(x), ld, static_cast<const bf16*>(y), ld,
                                       static_cast<const bf16*>(gate), static_cast<const bf16*>(shift),
                                       static_cast<const bf16*>(scale), ld_mod, sel, n_tokens, eps);
    return cudaGetLastError();
}

}  // namespace

bool adaln_warp_fits(sol_dtype dt, int64_t d)
{
    return dt == SOL_DTYPE_BF16 && d % 256 == 0 && d / 256 >= 1 && d / 256 <= 24;
}

bool prologue_regs_fits(sol_dtype dt, int64_t d)
{
    constexpr int W = SOL_PROLOGUE_REGS_WPR;
    return dt == SOL_DTYPE_BF16 && d % (256 * W) == 0 && d / (256 * W) >= 1 && d / (256 * W) <= 24 / W;
}

cudaError_t launch_prologue_regs(void* x_out, void* h, const void* x, const void* y, const void* gate,
                                 const void* shift, const void* scale, int64_t ld, int64_t ld_mod, const ModSel& sel,
                                 int64_t n_tokens, int64_t d, float eps, cudaStream_t s)
{
    constexpr int W = SOL_PROLOGUE_REGS_WPR;
    switch (d / (256 * W)) {
#define SOL_PRO_VPH(v)                                                                                           \
    case v:                                                                                                      \
        if constexpr (v * W <= 24) {                                                                             \
            if (y)                                                                                               \
                return launch_pro_vph<v, W, true>(x_out, h, x, y, gate, shift, scale, ld, ld_mod, sel, n_tokens, \
                                                  eps, s);                                                       \
            return launch_pro_vph<v, W, false>(x_out, h, x, y, gate, shift, scale, ld, ld_mod, sel, n_tokens,    \
                                               eps, s);                                                          \
        }                                                                                                        \
        break;
        SOL_PRO_VPH(1) SOL_PRO_VPH(2) SOL_PRO_VPH(3) SOL_PRO_VPH(4) SOL_PRO_VPH(5) SOL_PRO_VPH(6)
        SOL_PRO_VPH(7) SOL_PRO_VPH(8) SOL_PRO_VPH(9) SOL_PRO_VPH(10) SOL_PRO_VPH(11) SOL_PRO_VPH(12)
#undef SOL_PRO_VPH
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_adaln_warp(void* h, int64_t ld_h, const void* x, int64_t ld_x, const void* shift,
                              const void* scale, int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                              float eps, cudaStream_t s)
{
    switch (d / 256) {
#define SOL_ADALN_VPL(v) \
    case v: return launch_vpl<v>(h, ld_h, x, ld_x, shift, scale, ld_mod, sel, n_tokens, eps, s);
        SOL_ADALN_VPL(1) SOL_ADALN_VPL(2) SOL_ADALN_VPL(3) SOL_ADALN_VPL(4) SOL_ADALN_VPL(5) SOL_ADALN_VPL(6)
        SOL_ADALN_VPL(7) SOL_ADALN_VPL(8) SOL_ADALN_VPL(9) SOL_ADALN_VPL(10) SOL_ADALN_VPL(11) SOL_ADALN_VPL(12)
        SOL_ADALN_VPL(13) SOL_ADALN_VPL(14) SOL_ADALN_VPL(15) SOL_ADALN_VPL(16) SOL_ADALN_VPL(17) SOL_ADALN_VPL(18)
        SOL_ADALN_VPL(19) SOL_ADALN_VPL(20) SOL_ADALN_VPL(21) SOL_ADALN_VPL(22) SOL_ADALN_VPL(23) SOL_ADALN_VPL(24)
#undef SOL_ADALN_VPL
    }
    return cudaErrorInvalidValue;
}

}  // namespace sol
