// k_gemm.cu -- the block's linear layers y = a . W^T on the fifth-generation tensor
// cores, with the per-token operators fused into the operand load or the epilogue, so
// that their inputs and outputs never make an extra trip through HBM:
//   AdaLN -> QKV projection -> QK RMSNorm + 3D RoPE   (operand transform + epilogue)
//   MLP up projection -> SwiGLU                        (epilogue)
//   output / MLP down projection -> gated residual     (epilogue)
// [STM-RES] "SGLang acelera video do MiniMax-H3 em ate 6,2x em GPUs H200", section
// "Resultado principal": fused kernels cut memory traffic, intermediate tensors and
// launches without changing the math.
//
// Design (one persistent CTA per SM, 128 x 256 output tiles, K in steps of 64):
//   warp 0        tensor-copy producer: A tile 128 x 64 and B tile 256 x 64 (bf16,
//                 128-byte swizzle) per stage into a 4-stage shared-memory ring;
//   warp 1        MMA issuer: four 128 x 256 x 16 tcgen05.mma per stage into one of two
//                 TMEM accumulators (2 x 256 fp32 columns), so the epilogue of tile i
//                 overlaps the main loop of tile i+1; owns the TMEM allocation;
//   warps 2..5    epilogue: each thread owns one accumulator row (TMEM lane), reads it
//                 32 columns at a time and applies the fused operator;
//   warps 6..9    (AdaLN variant only) operand transform: rewrite each landed x tile in
//                 shared memory as h = (x - mean) * rstd * (1 + scale) + shift in bf16
//                 before the MMA reads it.
// Every wait on an mbarrier is bounded; a wait that gives up raises an error flag and
// the CTA drains its in-flight copies and MMAs, frees its TMEM and returns.
#include <algorithm>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace sol {
namespace gemm {

constexpr int BM = 128;                   // rows of a tile (TMEM lanes)
constexpr int BN = 256;                   // accumulator columns of a tile
constexpr int BK = 64;                    // K per stage: one 128-byte swizzle row of bf16
constexpr int UK = 16;                    // K of one tcgen05.mma (kind::f16)
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB
constexpr int B_BYTES = BN * BK * 2;      // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;         // two accumulators
constexpr int GROUP_M = 16;               // m-blocks per raster group (L2 reuse)
constexpr int PRODUCER_WARP = 0, MMA_WARP = 1, XFORM_WARP0 = 6;  // epilogue: warps 2..5
constexpr uint32_t kWaitLimit = 4096;     // polls of <= ~1 ms each

enum Epi : int { EPI_STORE = 0, EPI_GATED = 1, EPI_SWIGLU = 2, EPI_QKROPE = 3 };

// Shared-memory bookkeeping after the (1024-byte aligned) stage ring.
struct Bars {
    uint64_t full[STAGES];    // copy landed (tx count)
    uint64_t ready[STAGES];   // operand transformed (AdaLN variant), 128 arrivals
    uint64_t empty[STAGES];   // MMAs reading the stage finished (tcgen05.commit)
    uint64_t acc_full[2];     // accumulator complete (tcgen05.commit)
    uint64_t acc_empty[2];    // accumulator drained by the epilogue, 128 arrivals
    uint64_t drain;           // every MMA of this CTA finished (teardown)
    uint32_t tmem_base;
    volatile int32_t abort;
};

constexpr size_t smem_bytes() { return 1024 /*alignment slack*/ + (size_t)STAGES * STAGE_BYTES + sizeof(Bars); }

__device__ uint32_t g_gemm_error;

// Arguments of one launch (device pointers; sizes already validated on the host).
struct Params {
    int64_t M;            // rows (tokens)
    int32_t K;            // inner dimension, multiple of 64
    int32_t n_tiles_n;    // tiles along the output columns
    int32_t inner;        // SwiGLU: output width (B rows of the second half start here)
    int64_t num_tiles;
    bf16* out;
    int64_t ld_out;
    // gated residual
    const bf16* x;
    int64_t ld_x;
    const bf16* gate;
    // AdaLN operand transform
    const float2* stats;  // [M] (mean, rstd)
    const bf16* shift;
    const bf16* scale;
    int64_t ld_mod;
    ModSel sel;
    // QK RMSNorm + 3D RoPE epilogue
    const bf16* wq;
    const bf16* wk;
    const int32_t* pos;
    int32_t grid_H, grid_W;
    int64_t tps;          // tokens per sample for implicit positions (> 0)
    RopeDev rope;
    int32_t qk_cols;      // 2 * n_heads * head_dim: columns that get norm + RoPE
    float eps;
};

__device__ __forceinline__ void tile_coords(int64_t t, const Params& p, int64_t& m_blk, int32_t& n_blk)
{
    const int64_t num_m = (p.M + BM - 1) / BM;
    const int64_t per_group = (int64_t)GROUP_M * p.n_tiles_n;
    const int64_t g = t / per_group;
    const int64_t first_m = g * GROUP_M;
    const int64_t gm = min((int64_t)GROUP_M, num_m - first_m);
    const int64_t local = t - g * per_group;
    m_blk = first_m + local % gm;
    n_blk = (int32_t)(local / gm);
}

// Bounded wait that also gives up as soon as another role of the CTA has aborted.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, Bars* b)
{
    for (uint32_t i = 0; i < kWaitLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if (b->abort) return false;
    }
    return false;
}

__device__ __forceinline__ void raise_abort(Bars* b, uint32_t code)
{
    b->abort = 1;
    atomicOr(&g_gemm_error, code);
}

// ---------------------------------------------------------------------------------
// Producer: one thread streams the A and B tiles of every (tile, k-block) into the ring.
// B rows of a tile: [n0, n0+128) and [n1, n1+128); for SwiGLU n0 = 128*n_blk (gated
// half) and n1 = inner + 128*n_blk (multiplying half), otherwise n0 = 256*n_blk and
// n1 = n0 + 128.  Rows of A past M read as zeros (tensor-map bounds).
template <int EPI>
__device__ void run_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const Params& p, uint8_t* ring,
                             Bars* b)
{
    const int kblocks = p.K / BK;
    int s = 0;
    uint32_t phase = 0;
    int32_t last_parity[STAGES];
#pragma unroll
    for (int i = 0; i < STAGES; ++i) last_parity[i] = -1;

    for (int64_t t = blockIdx.x; t < p.num_tiles && !b->abort; t += gridDim.x) {
        int64_t m_blk;
        int32_t n_blk;
        tile_coords(t, p, m_blk, n_blk);
        const int32_t y_a = (int32_t)(m_blk * BM);
        const int32_t n0 = EPI == EPI_SWIGLU ? n_blk * (BN / 2) : n_blk * BN;
        const int32_t n1 = EPI == EPI_SWIGLU ? p.inner + n_blk * (BN / 2) : n0 + BN / 2;
        for (int kb = 0; kb < kblocks; ++kb) {
            if (!wait_or_abort(smem_u32(&b->empty[s]), phase ^ 1u, b)) {
                raise_abort(b, 1u);
                break;
            }
            const uint32_t full = smem_u32(&b->full[s]);
            const uint32_t dst = smem_u32(ring + (size_t)s * STAGE_BYTES);
            mbar_arrive_expect_tx(full, STAGE_BYTES);
            tc::tma_load_2d(dst, tmA, kb * BK, y_a, full);
            tc::tma_load_2d(dst + A_BYTES, tmB, kb * BK, n0, full);
            tc::tma_load_2d(dst + A_BYTES + B_BYTES / 2, tmB, kb * BK, n1, full);
            last_parity[s] = (int32_t)phase;
            if (++s == STAGES) {
                s = 0;
                phase ^= 1u;
            }
        }
    }
    // Teardown: every copy issued must have landed before the CTA may exit.
#pragma unroll
    for (int i = 0; i < STAGES; ++i)
        if (last_parity[i] >= 0 && !mbar_wait_bounded(smem_u32(&b->full[i]), (uint32_t)last_parity[i], kWaitLimit))
            atomicOr(&g_gemm_error, 2u);
}

// ---------------------------------------------------------------------------------
// MMA issuer: one thread.  Stage s is consumed once its copy landed (or, with the AdaLN
// transform, once the transform warps rewrote it); its slot is released by a commit
// when the four MMAs reading it finish.
template <bool PRO>
__device__ void run_mma(const Params& p, uint8_t* ring, Bars* b)
{
    const int kblocks = p.K / BK;
    const uint32_t idesc = tc::idesc_bf16_f32(BM, BN);
    int s = 0;
    uint32_t phase = 0;
    int64_t it = 0;
    for (int64_t t = blockIdx.x; t < p.num_tiles && !b->abort; t += gridDim.x, ++it) {
        const int ab = (int)(it & 1);
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        if (!wait_or_abort(smem_u32(&b->acc_empty[ab]), acc_phase ^ 1u, b)) {
            raise_abort(b, 4u);
            break;
        }
        tc::fence_after_sync();
        const uint32_t d_tmem = b->tmem_base + (uint32_t)(ab * BN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
            const uint32_t bar = PRO ? smem_u32(&b->ready[s]) : smem_u32(&b->full[s]);
            if (!wait_or_abort(bar, phase, b)) {
                raise_abort(b, 8u);
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const uint32_t a_addr = smem_u32(ring + (size_t)s * STAGE_BYTES);
            const uint64_t a_desc = tc::smem_desc_sw128(a_addr);
            const uint64_t b_desc = tc::smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk) {
                // advance K by 16 elements = 32 bytes inside the swizzle row (field >> 4)
                tc::mma_bf16(d_tmem, a_desc + (uint64_t)(kk * 2), b_desc + (uint64_t)(kk * 2), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
            }
            tc::commit(smem_u32(&b->empty[s]));
            if (++s == STAGES) {
                s = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        tc::commit(smem_u32(&b->acc_full[ab]));
    }
    // Teardown: wait for every MMA this thread issued.
    tc::commit(smem_u32(&b->drain));
    if (!mbar_wait_bounded(smem_u32(&b->drain), 0u, kWaitLimit)) atomicOr(&g_gemm_error, 16u);
}

// ---------------------------------------------------------------------------------
// Epilogue helpers.

// silu(a) * b with one ex2 and one reciprocal on the MUFU pipe (relative error a few
// 1e-7, far below a bf16 ulp); a very negative a gives 1/inf = 0, the limit -0.
__device__ __forceinline__ float silu_mul_fast(float a, float b)
{
    float e, r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-1.4426950408889634f * a));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + e));
    return a * r * b;
}

__device__ __forceinline__ void store32(bf16* dst, const float* v)
{
#pragma unroll
    for (int j = 0; j < 4; ++j) *reinterpret_cast<uint4*>(dst + 8 * j) = pack<bf16>(v + 8 * j);
}

// Token position (t, h, w) of `row`, clamped into the tables, as the per-token kernels
// take it: explicit pos[row], else the row-major grid of its sample.
__device__ __forceinline__ void token_pos(int64_t row, const Params& p, int& p0, int& p1, int& p2)
{
    if (p.pos) {
        p0 = min(max(__ldg(p.pos + 3 * row + 0), 0), p.rope.max[0] - 1);
        p1 = min(max(__ldg(p.pos + 3 * row + 1), 0), p.rope.max[1] - 1);
        p2 = min(max(__ldg(p.pos + 3 * row + 2), 0), p.rope.max[2] - 1);
    } else {
        const int64_t nl = row % p.tps;
        p0 = min((int)(nl / ((int64_t)p.grid_H * p.grid_W)), p.rope.max[0] - 1);
        p1 = min((int)((nl / p.grid_W) % p.grid_H), p.rope.max[1] - 1);
        p2 = min((int)(nl % p.grid_W), p.rope.max[2] - 1);
    }
}

// One 128-wide head vector of the accumulator row (TMEM columns taddr .. +127):
// v / sqrt(mean(v^2) + eps) * w, then the interleaved 3D rotation, stored to dst.
__device__ __forceinline__ void qk_head(uint32_t taddr, bool live, const bf16* w, const Params& p, int p0, int p1,
                                        int p2, bf16* dst)
{
    float v[32];
    float ss = 0.f;
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        tc::ld32(taddr + 32 * c, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);
    }
    const float r = rsqrtf(ss * (1.f / 128.f) + p.eps);
    const int h0 = p.rope.half[0], h01 = p.rope.half[0] + p.rope.half[1];
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
        tc::ld32(taddr + 32 * c, v);
        if (!live) continue;
        float fw[32];
        if (w) {
#pragma unroll
            for (int j = 0; j < 4; ++j) unpack<bf16>(ld_cached(w + 32 * c + 8 * j), fw + 8 * j);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) fw[i] = 1.f;
        }
        float o[32];
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const int pi = 16 * c + m;  // pair index inside the head
            const float2* tab;
            if (pi < h0)
                tab = p.rope.tab[0] + pi + (int64_t)p0 * p.rope.half[0];
            else if (pi < h01)
                tab = p.rope.tab[1] + (pi - h0) + (int64_t)p1 * p.rope.half[1];
            else
                tab = p.rope.tab[2] + (pi - h01) + (int64_t)p2 * p.rope.half[2];
            const float2 cs = __ldg(tab);
            const float a = v[2 * m] * r * fw[2 * m];
            const float b = v[2 * m + 1] * r * fw[2 * m + 1];
            o[2 * m] = a * cs.x - b * cs.y;
            o[2 * m + 1] = a * cs.y + b * cs.x;
        }
        store32(dst + 32 * c, o);
    }
}

// Epilogue warps 2..5: thread (warp w, lane l) owns accumulator row 32*(w % 4) + l, the
// TMEM lane quarter warp w may access.
template <int EPI>
__device__ void run_epilogue(const Params& p, Bars* b)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    int64_t it = 0;
    for (int64_t t = blockIdx.x; t < p.num_tiles; t += gridDim.x, ++it) {
        const int ab = (int)(it & 1);
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        const bool got = wait_or_abort(smem_u32(&b->acc_full[ab]), acc_phase, b);
        if (!__all_sync(0xffffffffu, got)) {
            raise_abort(b, 32u);
            break;
        }
        tc::fence_after_sync();
        int64_t m_blk;
        int32_t n_blk;
        tile_coords(t, p, m_blk, n_blk);
        const int64_t row = m_blk * BM + quarter * 32 + lane;
        const bool live = row < p.M;
        const uint32_t tbase = b->tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * BN);
        float v[32];

        if constexpr (EPI == EPI_STORE) {
            bf16* dst = p.out + row * p.ld_out + (int64_t)n_blk * BN;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                tc::ld32(tbase + 32 * c, v);
                        if (live) store32(dst + 32 * c, v);
            }
        } else if constexpr (EPI == EPI_GATED) {
            const int64_t col0 = (int64_t)n_blk * BN;
            const bf16* xr = p.x + row * p.ld_x + col0;
            const bf16* gr = nullptr;
            if (live && p.gate) gr = p.gate + mod_row(row, p.sel) * p.ld_mod + col0;
            bf16* dst = p.out + row * p.ld_out + col0;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                tc::ld32(tbase + 32 * c, v);
                        if (!live) continue;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float fx[8], fg[8];
                    unpack<bf16>(ld_plain(xr + 32 * c + 8 * j), fx);
                    if (gr) {
                        unpack<bf16>(ld_cached(gr + 32 * c + 8 * j), fg);
                    } else {
#pragma unroll
                        for (int e = 0; e < 8; ++e) fg[e] = 0.f;
                    }
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[8 * j + e] = fmaf(fg[e], v[8 * j + e], fx[e]);
                }
                store32(dst + 32 * c, v);
            }
        } else if constexpr (EPI == EPI_SWIGLU) {
            bf16* dst = p.out + row * p.ld_out + (int64_t)n_blk * (BN / 2);
            float u[32];
#pragma unroll 1
            for (int c = 0; c < BN / 64; ++c) {
                tc::ld32(tbase + 32 * c, v);
                tc::ld32(tbase + BN / 2 + 32 * c, u);
                        if (!live) continue;
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = silu_mul_fast(v[i], u[i]);
                store32(dst + 32 * c, v);
            }
        } else {  // EPI_QKROPE
            const int32_t col0 = n_blk * BN;
            bf16* dst = p.out + row * p.ld_out + col0;
            if (col0 >= p.qk_cols) {  // v heads: as projected
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    tc::ld32(tbase + 32 * c, v);
                                if (live) store32(dst + 32 * c, v);
                }
            } else {
                int p0 = 0, p1 = 0, p2 = 0;
                if (live) token_pos(row, p, p0, p1, p2);
                const bf16* w = col0 < p.qk_cols / 2 ? p.wq : p.wk;
                qk_head(tbase, live, w, p, p0, p1, p2, dst);
                qk_head(tbase + 128, live, w, p, p0, p1, p2, dst + 128);
            }
        }
        tc::fence_before_sync();
        tc::mbar_arrive(smem_u32(&b->acc_empty[ab]));
    }
}

// ---------------------------------------------------------------------------------
// AdaLN operand transform (warps 6..9): thread m rewrites row m of every landed A tile
// in place.  In the 128-byte swizzle a row is eight 16-byte chunks; physical chunk c of
// row m holds logical chunk c ^ (m % 8), i.e. columns 8*(c ^ (m % 8)) .. +7 of the
// k-block.  Thread m visits its chunks starting at chunk m % 8, so the eight threads of
// a quarter-warp touch eight different bank groups.  Rows past M stay zero (never
// stored).  Each thread fences its generic-proxy writes before arriving, so the
// tensor core (async proxy) reads the rewritten tile.
__device__ void run_transform(const Params& p, uint8_t* ring, Bars* b)
{
    const int m = threadIdx.x - XFORM_WARP0 * 32;
    const int kblocks = p.K / BK;
    int s = 0;
    uint32_t phase = 0;
    for (int64_t t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
        int64_t m_blk;
        int32_t n_blk;
        tile_coords(t, p, m_blk, n_blk);
        const int64_t row = m_blk * BM + m;
        const bool live = row < p.M;
        float mu = 0.f, rs = 0.f;
        const bf16 *sc = nullptr, *sh = nullptr;
        if (live) {
            const float2 st = __ldg(p.stats + row);
            mu = st.x;
            rs = st.y;
            const int64_t r = mod_row(row, p.sel);
            if (p.scale) sc = p.scale + r * p.ld_mod;
            if (p.shift) sh = p.shift + r * p.ld_mod;
        }
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
            if (!wait_or_abort(smem_u32(&b->full[s]), phase, b)) {
                raise_abort(b, 64u);
                ok = false;
                break;
            }
            if (live) {
                uint8_t* base = ring + (size_t)s * STAGE_BYTES + (size_t)m * 128;
#pragma unroll 2
                for (int i = 0; i < 8; ++i) {
                    const int c = (i + m) & 7;
                    const int k0 = kb * BK + 8 * (c ^ (m & 7));
                    uint4* cell = reinterpret_cast<uint4*>(base + 16 * c);
                    float2 f[4], g[4], h[4];
                    unpack2<bf16>(*cell, f);
                    if (sc) {
                        unpack2<bf16>(ld_cached(sc + k0), g);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) g[e] = make_float2(0.f, 0.f);
                    }
                    if (sh) {
                        unpack2<bf16>(ld_cached(sh + k0), h);
                    } else {
#pragma unroll
                        for (int e = 0; e < 4; ++e) h[e] = make_float2(0.f, 0.f);
                    }
                    const float2 mu2 = make_float2(mu, mu), rs2 = make_float2(rs, rs), one = make_float2(1.f, 1.f);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 nrm = __fmul2_rn(__fadd2_rn(f[e], make_float2(-mu2.x, -mu2.y)), rs2);
                        h[e] = __ffma2_rn(nrm, __fadd2_rn(one, g[e]), h[e]);
                    }
                    *cell = pack2<bf16>(h);
                }
            }
            fence_proxy_async_smem();
            tc::mbar_arrive(smem_u32(&b->ready[s]));
            if (++s == STAGES) {
                s = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
    }
}

// ---------------------------------------------------------------------------------
// The kernel: roles by warp (see the file header).
template <int EPI, bool PRO>
__global__ void __launch_bounds__(PRO ? 320 : 192, 1)
    k_linear(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Bars* b = reinterpret_cast<Bars*>(ring + (size_t)STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&b->full[i]), 1);
            mbar_init(smem_u32(&b->ready[i]), 128);
            mbar_init(smem_u32(&b->empty[i]), 1);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&b->acc_full[i]), 1);
            mbar_init(smem_u32(&b->acc_empty[i]), 128);
        }
        mbar_init(smem_u32(&b->drain), 1);
        b->abort = 0;
        mbar_fence_init();
        tc::prefetch_tmap(&tmA);
        tc::prefetch_tmap(&tmB);
    }
    if (warp == MMA_WARP) {
        tc::tmem_alloc(smem_u32(&b->tmem_base), TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    if (warp == PRODUCER_WARP) {
        if (lane == 0) run_producer<EPI>(&tmA, &tmB, p, ring, b);
    } else if (warp == MMA_WARP) {
        if (lane == 0) run_mma<PRO>(p, ring, b);
    } else if (warp < XFORM_WARP0) {
        run_epilogue<EPI>(p, b);
    } else if (PRO) {
        run_transform(p, ring, b);
    }

    tc::fence_before_sync();
    __syncthreads();
    if (warp == MMA_WARP) {
        tc::fence_after_sync();
        tc::tmem_dealloc(b->tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------------
// Row statistics for the AdaLN operand transform: (mean, 1/sqrt(var + eps)) of each row
// of x, biased variance by two passes (the second re-reads the row from L1/L2).  One
// warp per row.
__global__ void __launch_bounds__(256) k_row_stats(float2* stats, const bf16* x, int64_t ld_x, int64_t M, int32_t d,
                                                   float eps)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t wstep = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int nv = d / 8;
    for (int64_t row = w0; row < M; row += wstep) {
        const bf16* xr = x + row * ld_x;
        float s = 0.f;
        for (int v = lane; v < nv; v += 32) {
            float f[8];
            unpack<bf16>(ld_cached(xr + 8 * v), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) s += f[e];
        }
        const float mu = warp_sum(s) / (float)d;
        float q = 0.f;
        for (int v = lane; v < nv; v += 32) {
            float f[8];
            unpack<bf16>(ld_cached(xr + 8 * v), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float c = f[e] - mu;
                q = fmaf(c, c, q);
            }
        }
        const float var = warp_sum(q) / (float)d;
        if (lane == 0) stats[row] = make_float2(mu, rsqrtf(var + eps));
    }
}

}  // namespace gemm

// ---------------------------------------------------------------------------------
// Host side.

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            f = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }();
    return fn;
}

// 2-D bf16 tensor map over rows x cols (row stride ld elements), boxes of 64 columns x
// 128 rows in the 128-byte swizzle; out-of-range rows read as zeros.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {ld * 2};
    const cuuint32_t box[2] = {(cuuint32_t)gemm::BK, (cuuint32_t)(gemm::BM)};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool PRO>
cudaError_t launch_kernel(const CUtensorMap& ma, const CUtensorMap& mb, const gemm::Params& p, cudaStream_t s)
{
    auto kern = gemm::k_linear<EPI, PRO>;
    const size_t smem = gemm::smem_bytes();
    static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (attr != cudaSuccess) return attr;
    const int64_t grid = std::min<int64_t>(p.num_tiles, (int64_t)sm_count());
    kern<<<(unsigned)grid, PRO ? 320 : 192, smem, s>>>(ma, mb, p);
    return cudaGetLastError();
}

}  // namespace

size_t linear_smem_bytes() { return gemm::smem_bytes(); }

cudaError_t launch_linear(LinearEpi epi, bool adaln, const LinearLaunch& a, cudaStream_t s)
{
    if (a.M == 0) return cudaSuccess;
    CUtensorMap ma, mb;
    if (!make_map(&ma, a.a, (uint64_t)a.M, (uint64_t)a.K, (uint64_t)a.ld_a) ||
        !make_map(&mb, a.w, (uint64_t)a.N, (uint64_t)a.K, (uint64_t)a.ld_w)) {
        record_error("tensor map encoding failed (cuTensorMapEncodeTiled unavailable or refused the layout)");
        return cudaErrorInvalidValue;
    }
    gemm::Params p{};
    p.M = a.M;
    p.K = a.K;
    p.n_tiles_n = a.N / gemm::BN;  // SwiGLU: inner / 128 pair tiles of 256 columns
    p.inner = a.N / 2;
    p.num_tiles = (a.M + gemm::BM - 1) / gemm::BM * (int64_t)p.n_tiles_n;
    p.out = static_cast<bf16*>(a.out);
    p.ld_out = a.ld_out;
    p.x = static_cast<const bf16*>(a.x);
    p.ld_x = a.ld_x;
    p.gate = static_cast<const bf16*>(a.gate);
    p.stats = static_cast<const float2*>(a.stats);
    p.shift = static_cast<const bf16*>(a.shift);
    p.scale = static_cast<const bf16*>(a.scale);
    p.ld_mod = a.ld_mod;
    if (a.sel) p.sel = *a.sel;
    p.wq = static_cast<const bf16*>(a.wq);
    p.wk = static_cast<const bf16*>(a.wk);
    p.pos = a.pos;
    p.grid_H = a.grid_H;
    p.grid_W = a.grid_W;
    p.tps = a.tps > 0 ? a.tps : a.M;
    p.rope = a.rope;
    p.qk_cols = a.qk_cols;
    p.eps = a.eps;

    if (adaln) {
        const int64_t blocks = std::min<int64_t>((a.M + 7) / 8, (int64_t)sm_count() * 16);
        gemm::k_row_stats<<<(unsigned)blocks, 256, 0, s>>>(static_cast<float2*>(a.stats),
                                                           static_cast<const bf16*>(a.a), a.ld_a, a.M, a.K, a.eps);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    switch (epi) {
    case LINEAR_STORE:
        return adaln ? launch_kernel<gemm::EPI_STORE, true>(ma, mb, p, s) : launch_kernel<gemm::EPI_STORE, false>(ma, mb, p, s);
    case LINEAR_GATED:
        return launch_kernel<gemm::EPI_GATED, false>(ma, mb, p, s);
    case LINEAR_SWIGLU:
        return launch_kernel<gemm::EPI_SWIGLU, false>(ma, mb, p, s);
    case LINEAR_QKROPE:
        return adaln ? launch_kernel<gemm::EPI_QKROPE, true>(ma, mb, p, s)
                     : launch_kernel<gemm::EPI_QKROPE, false>(ma, mb, p, s);
    }
    return cudaErrorInvalidValue;
}

uint32_t gemm_device_error(bool clear)
{
    uint32_t v = 0;
    cudaMemcpyFromSymbol(&v, gemm::g_gemm_error, sizeof(v));
    if (clear) {
        const uint32_t z = 0;
        cudaMemcpyToSymbol(gemm::g_gemm_error, &z, sizeof(z));
    }
    return v;
}

}  // namespace sol
