// common.cuh -- device helpers shared by the libsol kernels: 16-byte vector I/O with
// cache hints, bf16/f32 <-> fp32 register conversion, modulation-row selection and
// block/segment reductions.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sol {

using bf16 = __nv_bfloat16;

// Elements of T in one 16-byte vector.
template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int N = 4; };
template <> struct Vec<bf16> { static constexpr int N = 8; };

// Streaming load / store of data touched once (evict-first in L1 and L2) and a
// read-only cached load for small tensors every CTA re-reads (modulation rows, weights).
__device__ __forceinline__ uint4 ld_stream(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ uint4 ld_cached(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void st_stream(void* p, const uint4& v) { __stcs(reinterpret_cast<uint4*>(p), v); }

// Widen one 16-byte vector to fp32.  bf16 -> fp32 is exact: the bf16 bits are the high
// half of the binary32 with the same value.
template <typename T> __device__ __forceinline__ void unpack(const uint4& r, float* f);
template <> __device__ __forceinline__ void unpack<float>(const uint4& r, float* f)
{
    f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
}
template <> __device__ __forceinline__ void unpack<bf16>(const uint4& r, float* f)
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Narrow fp32 registers to one 16-byte vector, rounding to nearest even.
template <typename T> __device__ __forceinline__ uint4 pack(const float* f);
template <> __device__ __forceinline__ uint4 pack<float>(const float* f)
{
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
}
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi)
{
    __nv_bfloat162 b = __float22bfloat162_rn(make_float2(lo, hi));
    return *reinterpret_cast<uint32_t*>(&b);
}
template <> __device__ __forceinline__ uint4 pack<bf16>(const float* f)
{
    return make_uint4(pack2_bf16(f[0], f[1]), pack2_bf16(f[2], f[3]), pack2_bf16(f[4], f[5]),
                      pack2_bf16(f[6], f[7]));
}

// Modulation-row selection for packed multi-sample, multi-stream sequences.
struct ModSel {
    const uint8_t* stream_id;   // [n_tokens] or nullptr
    int32_t n_streams;          // >= 1
    int64_t tokens_per_sample;  // > 0, or 0 = one sample
};

__device__ __forceinline__ int64_t mod_row(int64_t n, const ModSel& m)
{
    const int64_t sample = m.tokens_per_sample > 0 ? n / m.tokens_per_sample : 0;
    int32_t s = 0;
    if (m.stream_id) {
        s = m.stream_id[n];
        if (s >= m.n_streams) s = m.n_streams - 1;
    }
    return sample * m.n_streams + s;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Sum over the CTA; every thread gets the total.  `buf` holds one float per warp and
// must not be reused before the next __syncthreads() that every thread passes after
// reading it (callers alternate two buffers).
__device__ __forceinline__ float block_sum(float v, float* buf)
{
    v = warp_sum(v);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) buf[warp] = v;
    __syncthreads();
    const int nw = blockDim.x >> 5;
    float t = 0.f;
    for (int i = 0; i < nw; ++i) t += buf[i];
    return t;
}

}  // namespace sol
