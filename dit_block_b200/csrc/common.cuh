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

// 16-byte loads and stores of data touched once:
//   ld_stream     ld.global.cs (evict first) -- for inputs the same kernel may overwrite
//                 in place (each element is read once, before its owner writes it);
//   ld_stream_ro  ld.global.nc (read-only path) -- for inputs nothing in the kernel writes;
//   st_stream     st.global.L1::no_allocate -- outputs are never re-read by the kernel.
// ld_cached: read-only cached load for small tensors every CTA re-reads (modulation
// rows, weights).  The forms were chosen by timing each op on B200.
__device__ __forceinline__ uint4 ld_stream(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ uint4 ld_stream_ro(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ uint4 ld_cached(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
// default-policy load, for data the kernel reads again shortly (kept in L2)
__device__ __forceinline__ uint4 ld_plain(const void* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void st_stream(void* p, const uint4& v)
{
    asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

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

// Widen / narrow one 16-byte vector as fp32 pairs, for the packed f32x2 arithmetic of
// sm_100 (__fadd2_rn, __fmul2_rn, __ffma2_rn: two IEEE fp32 operations per instruction).
template <typename T> __device__ __forceinline__ void unpack2(const uint4& r, float2* f);
template <> __device__ __forceinline__ void unpack2<float>(const uint4& r, float2* f)
{
    f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    f[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
}
template <> __device__ __forceinline__ void unpack2<bf16>(const uint4& r, float2* f)
{
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}
template <typename T> __device__ __forceinline__ uint4 pack2(const float2* f);
template <> __device__ __forceinline__ uint4 pack2<float>(const float2* f)
{
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
}
template <> __device__ __forceinline__ uint4 pack2<bf16>(const float2* f)
{
    return make_uint4(pack2_bf16(f[0].x, f[0].y), pack2_bf16(f[1].x, f[1].y), pack2_bf16(f[2].x, f[2].y),
                      pack2_bf16(f[3].x, f[3].y));
}

// Modulation-row selection for packed multi-sample, multi-stream sequences.
// The sample index n / tokens_per_sample uses a precomputed multiply-and-shift
// (division by an invariant integer, Granlund and Montgomery 1994) when every token
// index is below 2^31: q = (umulhi(n, m) + n) >> s with s = ceil(log2 d) and
// m = floor(2^32 * (2^s - d) / d) + 1; otherwise a plain 64-bit division.
struct ModSel {
    const uint8_t* stream_id;   // [n_tokens] or nullptr
    int32_t n_streams;          // >= 1
    int64_t tokens_per_sample;  // > 0, or 0 = one sample
    uint32_t div_m;             // multiplier for the 32-bit fast path
    uint32_t div_s;             // shift for the 32-bit fast path
    int32_t div_fast;           // 1: use the fast path
};

// Host side: fill the fast-division fields for `n_tokens` tokens.
inline void modsel_prepare(ModSel& m, int64_t n_tokens)
{
    m.div_fast = 0;
    m.div_m = 0;
    m.div_s = 0;
    const int64_t d = m.tokens_per_sample;
    if (d <= 0 || d >= (int64_t)1 << 31 || n_tokens >= (int64_t)1 << 31) return;
    uint32_t s = 0;
    while (((uint64_t)1 << s) < (uint64_t)d) ++s;
    const uint64_t two32 = (uint64_t)1 << 32;
    m.div_m = (uint32_t)((two32 * (((uint64_t)1 << s) - (uint64_t)d)) / (uint64_t)d + 1);
    m.div_s = s;
    m.div_fast = 1;
}

// Sample index of token n (0 when the call is one sample).
__device__ __forceinline__ int64_t sample_of(int64_t n, const ModSel& m)
{
    if (m.tokens_per_sample <= 0) return 0;
    if (m.div_fast) {
        const uint32_t nn = (uint32_t)n;
        return (int64_t)((__umulhi(nn, m.div_m) + nn) >> m.div_s);
    }
    return n / m.tokens_per_sample;
}

__device__ __forceinline__ int64_t mod_row(int64_t n, const ModSel& m)
{
    int64_t sample = 0;
    if (m.tokens_per_sample > 0) {
        if (m.div_fast) {
            const uint32_t nn = (uint32_t)n;
            sample = (int64_t)((__umulhi(nn, m.div_m) + nn) >> m.div_s);
        } else {
            sample = n / m.tokens_per_sample;
        }
    }
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

// ---------------------------------------------------------------------------------
// Bulk asynchronous copies (global -> this CTA's shared memory) completed on an mbarrier.
namespace sol {

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make initialised mbarriers visible to the async proxy before the first bulk copy.
__device__ __forceinline__ void mbar_fence_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// One bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
// from global memory into this CTA's shared memory, counted on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before its later
// async-proxy ones (a bulk copy refilling a buffer other threads just read).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One poll of phase `parity`; a thread whose phase is not complete may be suspended for
// up to ~1 ms (the hint, in ns) instead of spinning, so waiting warps leave the issue
// slots to the warps that have work.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}

// Wait for phase `parity` of `bar` to complete, giving up after `limit` polls (each poll
// suspends for at most about a millisecond).  Returns false on give-up.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint32_t limit)
{
    for (uint32_t i = 0; i < limit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

}  // namespace sol
