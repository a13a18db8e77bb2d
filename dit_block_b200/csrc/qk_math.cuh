// qk_math.cuh -- the per-slot arithmetic of QK RMSNorm + interleaved 3D RoPE shared by the
// staged kernels (k_qk_cta.cu: the epilogue and the epilogue with block means) and the
// row-in-registers kernel (k_qk_regs.cu), whose in-place results must be the same bits.
//
// A lane holds 8 consecutive elements (4 interleaved rotary pairs) of a head vector; its
// RMSNorm weights w[0..7] and its pairs' (cos, sin) are fixed for the row, so the weights
// are folded into the rotation once per row:
//     o_2m   = (v_2m r) w_2m c_m - (v_2m+1 r) w_2m+1 s_m
//     o_2m+1 = (v_2m r) w_2m s_m + (v_2m+1 r) w_2m+1 c_m
// with r = 1 / sqrt(mean(v^2) + eps) of the head vector -- the same value as normalising,
// weighting and rotating in turn, in fewer instructions per element (the products with r
// are packed f32x2 multiplies).
#pragma once

#include "common.cuh"

namespace sol {

// Rotation coefficients of one row: kc[4m..4m+3] = (w_2m c_m, w_2m+1 s_m, w_2m s_m, w_2m+1 c_m).
__device__ __forceinline__ void qk_coefs(const float (&w)[8], const float (&cs)[4], const float (&sn)[4],
                                         float (&kc)[16])
{
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        kc[4 * m + 0] = w[2 * m] * cs[m];
        kc[4 * m + 1] = w[2 * m + 1] * sn[m];
        kc[4 * m + 2] = w[2 * m] * sn[m];
        kc[4 * m + 3] = w[2 * m + 1] * cs[m];
    }
}

// Sum of squares of a lane's 8 elements (as 4 pairs).
__device__ __forceinline__ float qk_sumsq(const float2 (&f)[4])
{
    float2 a = __fmul2_rn(f[0], f[0]);
#pragma unroll
    for (int m = 1; m < 4; ++m) a = __ffma2_rn(f[m], f[m], a);
    return a.x + a.y;
}

// The lane's 8 outputs of a head vector with 1 / rms r.
__device__ __forceinline__ void qk_rotate(const float2 (&f)[4], float r, const float (&kc)[16], float (&o)[8])
{
    const float2 r2 = make_float2(r, r);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float2 v = __fmul2_rn(f[m], r2);
        o[2 * m] = fmaf(v.x, kc[4 * m + 0], -(v.y * kc[4 * m + 1]));
        o[2 * m + 1] = fmaf(v.x, kc[4 * m + 2], v.y * kc[4 * m + 3]);
    }
}

}  // namespace sol
