// k_qk_regs.cu -- QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合"]
// (bf16, head_dim 128) with one warp per (token, q or k) row held in registers.
//
// Lane l holds 16-byte vectors l, l + 32, ..., of the row (VPL of them: n_heads * 128 =
// 256 * VPL), so register slot i of lanes 0..15 / 16..31 is exactly head vector 2i /
// 2i + 1, and every lane owns the same 8-element slice (elements 8 * (l % 16) ..) of
// every head vector.  So:
//   * its RMSNorm weights and its four rotary pairs' (cos, sin) are loaded once per row
//     (the pairs' axis and frequency never change; only the token's position does);
//   * the VPL head vectors' RMS reductions are VPL independent xor-shuffle trees over
//     half-warps, which the compiler interleaves (no dependent chain per head);
//   * all VPL loads are in flight before any is used, and the row is written only after
//     it was read completely (in place is safe).
// Arithmetic is fp32: v / sqrt(mean(v^2) + eps) * w, then the interleaved rotation of
// pairs (2j, 2j + 1), as the per-step kernel (k_qk.cu) computes it.  The staged kernel of
// k_qk_cta.cu takes the same shapes when q and k are both given; this one serves the calls
// with q or k alone.
#include <algorithm>

#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "qk_math.cuh"

// Launch shape: blocks of 64 threads, >= 4 per SM (the row needs ~200 registers per lane
// unspilled; the same shape as the AdaLN row kernel).
#ifndef SOL_QK_REGS_BLOCK
#define SOL_QK_REGS_BLOCK 64
#endif
#ifndef SOL_QK_REGS_MINB
#define SOL_QK_REGS_MINB 4
#endif


namespace sol {

template <int VPL>
__global__ void __launch_bounds__(SOL_QK_REGS_BLOCK, SOL_QK_REGS_MINB)
    k_qk_regs(bf16* q_out, bf16* k_out, int64_t ld_qo, int64_t ld_ko, const bf16* q, const bf16* k, int64_t ld_q,
              int64_t ld_k, const bf16* __restrict__ wq, const bf16* __restrict__ wk, const int32_t* __restrict__ pos,
              int32_t grid_H, int32_t grid_W, int64_t tokens_per_sample, RopeDev rope, int64_t n_tokens, float eps)
{
    const int lane = threadIdx.x & 31;
    const int sub = lane & 15;  // element slice 8 * sub .. + 7 of every head vector
    float fwq[8], fwk[8];
    if (wq) {
        unpack<bf16>(ld_cached(wq + 8 * sub), fwq);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) fwq[e] = 1.f;
    }
    if (wk) {
        unpack<bf16>(ld_cached(wk + 8 * sub), fwk);
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) fwk[e] = 1.f;
    }
    // this lane's four rotary pairs: axis, table column, row stride
    const float2* tb[4];
    int stride[4], axis[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int pi = 4 * sub + m;
        const int h0 = rope.half[0], h01 = rope.half[0] + rope.half[1];
        axis[m] = pi < h0 ? 0 : (pi < h01 ? 1 : 2);
        tb[m] = axis[m] == 0 ? rope.tab[0] + pi : (axis[m] == 1 ? rope.tab[1] + (pi - h0) : rope.tab[2] + (pi - h01));
        stride[m] = axis[m] == 0 ? rope.half[0] : (axis[m] == 1 ? rope.half[1] : rope.half[2]);
    }

    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t wstep = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t item = w0; item < 2 * n_tokens; item += wstep) {
        const int64_t n = item >> 1;
        const int isk = (int)(item & 1);
        const bf16* src = isk ? k : q;
        if (!src) continue;  // uniform over the warp
        src += n * (isk ? ld_k : ld_q) + 8 * lane;
        uint4 xv[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) xv[i] = ld_stream(src + 256 * i);

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
        float cs[4], sn[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int pm = axis[m] == 0 ? p0 : (axis[m] == 1 ? p1 : p2);
            const float2 t = __ldg(tb[m] + (int64_t)pm * stride[m]);
            cs[m] = t.x;
            sn[m] = t.y;
        }
        float w[8];  // selects, not an indexed array (which would live in local memory)
#pragma unroll
        for (int e = 0; e < 8; ++e) w[e] = isk ? fwk[e] : fwq[e];
        float kc[16];  // weights folded into the rotation once per row
        qk_coefs(w, cs, sn, kc);
        bf16* dst = (isk ? k_out + n * ld_ko : q_out + n * ld_qo) + 8 * lane;

        // GS slots at a time: widen once, sums of squares, GS independent half-warp trees,
        // then normalise, rotate and store them
        constexpr int GS = 4;
#pragma unroll
        for (int i0 = 0; i0 < VPL; i0 += GS) {
            float2 f[GS][4];
            float ss[GS];
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                ss[u] = 0.f;
                if (i0 + u < VPL) {
                    unpack2<bf16>(xv[i0 + u], f[u]);
                    ss[u] = qk_sumsq(f[u]);
                }
            }
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) {
#pragma unroll
                for (int u = 0; u < GS; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], off);
            }
#pragma unroll
            for (int u = 0; u < GS; ++u) {
                if (i0 + u < VPL) {
                    float o[8];
                    qk_rotate(f[u], rsqrtf(ss[u] * (1.f / 128.f) + eps), kc, o);
                    st_stream(dst + 256 * (i0 + u), pack<bf16>(o));
                }
            }
        }
    }
}

namespace {

template <int VPL>
cudaError_t launch_vpl(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                       int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                       int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens, float eps, cudaStream_t s)
{
    auto kern = k_qk_regs<VPL>;
    constexpr int block = SOL_QK_REGS_BLOCK;
    const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), block, 0);
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t grid = std::min<int64_t>((int64_t)per_sm * sm_count(), (2 * n_tokens + block / 32 - 1) / (block / 32));
    kern<<<(unsigned)grid, block, 0, s>>>(static_cast<bf16*>(q_out), static_cast<bf16*>(k_out), ld_qo, ld_ko,
                                        static_cast<const bf16*>(q), static_cast<const bf16*>(k), ld_q, ld_k,
                                        static_cast<const bf16*>(wq), static_cast<const bf16*>(wk), pos, grid_H,
                                        grid_W, tps, rope, n_tokens, eps);
    return cudaGetLastError();
}

}  // namespace

bool qk_regs_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim)
{
    return dt == SOL_DTYPE_BF16 && head_dim == 128 && n_heads % 2 == 0 && n_heads >= 2 && n_heads <= 48;
}

cudaError_t launch_qk_regs(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                           int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                           int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                           int32_t n_heads, float eps, cudaStream_t s)
{
    switch (n_heads / 2) {
#define SOL_QK_VPL(v)                                                                                              \
    case v:                                                                                                        \
        return launch_vpl<v>(q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos, grid_H, grid_W, tps, rope, \
                             n_tokens, eps, s);
        SOL_QK_VPL(1) SOL_QK_VPL(2) SOL_QK_VPL(3) SOL_QK_VPL(4) SOL_QK_VPL(5) SOL_QK_VPL(6) SOL_QK_VPL(7)
        SOL_QK_VPL(8) SOL_QK_VPL(9) SOL_QK_VPL(10) SOL_QK_VPL(11) SOL_QK_VPL(12) SOL_QK_VPL(13) SOL_QK_VPL(14)
        SOL_QK_VPL(15) SOL_QK_VPL(16) SOL_QK_VPL(17) SOL_QK_VPL(18) SOL_QK_VPL(19) SOL_QK_VPL(20)
        SOL_QK_VPL(21) SOL_QK_VPL(22) SOL_QK_VPL(23) SOL_QK_VPL(24)
#undef SOL_QK_VPL
    }
    return cudaErrorInvalidValue;
}

}  // namespace sol
