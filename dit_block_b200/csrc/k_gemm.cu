// k_gemm.cu -- the block's linear layers y = a . W^T on the fifth-generation tensor
// cores, with the per-token operators fused in, so that their inputs and outputs never
// make an extra trip through HBM:
//   AdaLN -> QKV projection -> QK RMSNorm + 3D RoPE   (AdaLN strategy + epilogue)
//   AdaLN -> MLP up projection -> SwiGLU              (AdaLN strategy + epilogue)
//   MLP up projection -> SwiGLU                        (epilogue)
//   output / MLP down projection -> gated residual     (epilogue)
// [STM-RES] "SGLang acelera video do MiniMax-H3 em ate 6,2x em GPUs H200", section
// "Resultado principal": fused kernels cut memory traffic, intermediate tensors and
// launches without changing the math.
//
// Design: persistent CTAs, output tiles of 256 accumulator columns, K in steps of 64
// (one 128-byte swizzle row of bf16).  Two shapes of the same kernel:
//   single  one CTA per SM, 128 x 256 tiles, 4-stage ring of A 128x64 + B 256x64;
//   pair    a cluster of two CTAs on two SMs, 256 x 256 tiles computed by 256-row
//           tcgen05.mma (cta_group::2) issued by the leader CTA; each CTA loads half
//           of A (its 128 rows) and half of B (128 of the 256 columns) into a 7-stage
//           ring of 32 KiB stages and holds its 128 accumulator rows in its own TMEM.
//           Per SM the copies per MMA drop by a third and the ring is half as deep
//           again, which hides the copy latency.  The variant with the AdaLN operand
//           transform runs single (see use_pair()).
// AdaLN, three ways (the caller's sol_adaln_strategy): "stage" stages h = AdaLN(x) through the
// workspace with the per-token row kernel and runs the plain GEMM on it (one h round
// trip, measured fastest); "fold" folds (1 + scale) into a per-call copy of the weights
// and corrects each accumulator row as rstd * (acc - mean * c_r) + b_r in the epilogue (a
// plain GEMM on the raw tokens; see k_fold_weights); "transform" rewrites each landed x
// tile in shared memory as h before the MMA reads it (the operand transform).
// Warp roles:
//   warp 0        tensor-copy producer (one thread);
//   warp 1        MMA issuer (one thread; the leader CTA only in a pair) into one of two
//                 TMEM accumulators of 256 fp32 columns, so the epilogue of tile i
//                 overlaps the main loop of tile i+1; owns the TMEM allocation;
//   warps 2..9    epilogue (2..5 for the plain and gated-residual epilogues and beside
//                 the transform): each thread owns one accumulator row (TMEM lane) and
//                 half of its columns (all of them with four warps), reads them 32
//                 columns at a time and applies the operator;
//   warps 6..13   (operand-transform variant only) two groups on alternate stages.
// Every copy lands in the shared memory of the one CTA that issued it, and the leader
// commits to its own and to the peer's barriers one at a time.  Every wait on an mbarrier
// is bounded; a wait that gives up raises an error flag and the CTA drains its in-flight
// copies and MMAs, frees its TMEM and returns.
#include <algorithm>
#include <mutex>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace sol {
namespace gemm {

constexpr int BM = 128;                   // accumulator rows per CTA (TMEM lanes)
constexpr int BN = 256;                   // accumulator columns of a tile
constexpr int BK = 64;                    // K per stage
constexpr int UK = 16;                    // K of one tcgen05.mma (kind::f16)
constexpr int A_BYTES = BM * BK * 2;      // 16 KiB: this CTA's rows of A per stage
constexpr int TMEM_COLS = 2 * BN;         // two accumulators
#ifndef SOL_GEMM_GROUP_M
#define SOL_GEMM_GROUP_M 16
#endif
#ifndef SOL_GEMM_PAIR_STAGES
#define SOL_GEMM_PAIR_STAGES 7
#endif
constexpr int GROUP_M = SOL_GEMM_GROUP_M;  // m-blocks per raster group (L2 reuse)
constexpr int MAX_STAGES = SOL_GEMM_PAIR_STAGES > 4 ? SOL_GEMM_PAIR_STAGES : 4;
constexpr int PRODUCER_WARP = 0, MMA_WARP = 1, EPI_WARP0 = 2, XFORM_WARP0 = 6;
constexpr uint32_t kWaitLimit = 4096;     // polls of <= ~1 ms each

template <bool PAIR> struct Shape {
    static constexpr int STAGES = PAIR ? SOL_GEMM_PAIR_STAGES : 4;
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;   // rows of B (output columns) this CTA loads
    static constexpr int B_BYTES = B_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int TILE_M = PAIR ? 2 * BM : BM;   // rows of one output tile
};

enum Epi : int { EPI_STORE = 0, EPI_GATED = 1, EPI_SWIGLU = 2, EPI_QKROPE = 3 };

// Epilogue warps: one per TMEM lane quarter for the plain and gated-residual epilogues (each
// takes all 256 columns of its 32 rows), two per quarter (a column half each) for SwiGLU and
// the QK norm + RoPE, whose arithmetic per element is larger, and 4 beside the AdaLN
// transform warps (the register file holds no more).  Measured at 32,768 tokens on B200:
// O projection + gated residual 1.47-1.51 ms with 8 warps, 1.18-1.24 with 4; the bare QKV
// GEMM 3.81-3.92 / 3.69-3.74 ms; QKV + QK norm + RoPE 4.45 / 4.90-5.05 ms; up projection +
// SwiGLU 6.69-6.93 / 6.90-7.01 ms.  Fewer epilogue warps disturb the copies and the MMA
// less while the accumulator hand-over still keeps up.
template <int EPI, bool PRO> __host__ __device__ constexpr int epi_warps()
{
    return PRO ? 4 : ((EPI == EPI_STORE || EPI == EPI_GATED) ? 4 : 8);
}

// Shared-memory bookkeeping after the (1024-byte aligned) stage ring.  The barriers the
// MMA waits on live in the leader: full (the copies of both CTAs of a pair, armed by the
// leader alone), ready (transforms of both CTAs), acc_empty (epilogues of both CTAs).
// With the AdaLN transform each CTA's copies complete on its own full[s], which its
// transform warps wait for.
struct Bars {
    uint64_t full[MAX_STAGES];       // copies landed (tx count)
    uint64_t ready[MAX_STAGES];      // A rewritten by the transform, one arrival per warp
    uint64_t empty[MAX_STAGES];      // MMAs reading the stage finished (tcgen05.commit)
    uint64_t acc_full[2];            // accumulator complete (tcgen05.commit)
    uint64_t acc_empty[2];           // accumulator drained, one arrival per epilogue warp
    uint64_t drain;                  // every MMA issued by this CTA finished (teardown)
    int32_t peer_last[MAX_STAGES];   // pair leader: phase of the peer's last copy per stage (-1: none)
    uint32_t tmem_base;
    volatile int32_t abort;
};

template <bool PAIR> constexpr size_t smem_bytes()
{
    return 1024 /*alignment slack*/ + (size_t)Shape<PAIR>::STAGES * Shape<PAIR>::STAGE_BYTES + sizeof(Bars);
}

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
    // AdaLN (both strategies)
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
    // AdaLN folded into the weights: y = rstd * (x . V_r^T - mean * c_r) + b_r
    const uint32_t* rmask;  // [ceil(M / 128)]: bit r set if a row of the 128-row block uses row r
    const float* fold_c;    // [R, n_w]: column sums of the folded weights V_r
    const float* fold_b;    // [R, n_w]: shift_r . W^T
    int32_t n_w;            // output columns (rows of W) per modulation row
};

// Where this CTA sits: its rank in the pair (0 when single), the index of its pair (or
// CTA) among the persistent workers, and how many workers there are.
struct Where {
    uint32_t rank;
    int64_t worker, n_workers;
};

template <bool PAIR> __device__ __forceinline__ Where where()
{
    Where w;
    w.rank = PAIR ? tc::cluster_rank() : 0u;
    w.worker = PAIR ? blockIdx.x / 2 : blockIdx.x;
    w.n_workers = PAIR ? gridDim.x / 2 : gridDim.x;
    return w;
}

// Tile t -> (m-block of TILE_M rows, n-block of 256 columns), rastered in groups of
// GROUP_M m-blocks so concurrent tiles share A rows and B columns in L2.
template <bool PAIR>
__device__ __forceinline__ void tile_coords(int64_t t, const Params& p, int64_t& m_blk, int32_t& n_blk)
{
    const int64_t num_m = (p.M + Shape<PAIR>::TILE_M - 1) / Shape<PAIR>::TILE_M;
    const int64_t per_group = (int64_t)GROUP_M * p.n_tiles_n;
    const int64_t g = t / per_group;
    const int64_t first_m = g * GROUP_M;
    const int64_t gm = min((int64_t)GROUP_M, num_m - first_m);
    const int64_t local = t - g * per_group;
    m_blk = first_m + local % gm;
    n_blk = (int32_t)(local / gm);
}

// Modulation rows used by the rows of m-block m_blk (AdaLN fold), else one pass.
template <bool PAIR, bool FOLD>
__device__ __forceinline__ uint32_t tile_rows_mask(const Params& p, int64_t m_blk)
{
    if (!FOLD) return 1u;
    const int64_t b0 = m_blk * (Shape<PAIR>::TILE_M / BM);
    uint32_t m = __ldg(p.rmask + b0);
    if (PAIR && (b0 + 1) * BM < p.M) m |= __ldg(p.rmask + b0 + 1);
    return m;
}

// One unit of work: a tile or, with the AdaLN fold, a tile and one modulation row present
// in its rows (computed with that row's folded weights; the epilogue stores only the rows
// that use it).  Every role walks the same sequence of passes.
struct Pass {
    int64_t t;
    int64_t m_blk;
    int32_t n_blk;
    uint32_t rm;  // modulation rows of this tile still to do
    int32_t r;    // modulation row of this pass
};

__device__ __forceinline__ Pass pass_begin() { return Pass{-1, 0, 0, 0u, 0}; }

template <bool PAIR, bool FOLD>
__device__ __forceinline__ bool next_pass(Pass& q, const Params& p, const Where& w)
{
    while (true) {
        if (q.rm) {
            q.r = __ffs(q.rm) - 1;
            q.rm &= q.rm - 1;
            return true;
        }
        q.t = q.t < 0 ? w.worker : q.t + w.n_workers;
        if (q.t >= p.num_tiles) return false;
        tile_coords<PAIR>(q.t, p, q.m_blk, q.n_blk);
        q.rm = tile_rows_mask<PAIR, FOLD>(p, q.m_blk);
    }
}

// Bounded wait that also gives up as soon as another role of the CTA has aborted.
// Pair barriers are waited with acquire at cluster scope (the peer arrives on them).
// SOL_GEMM_PAIR_POLL 1: pair waits poll with the hardware's own short time limit (no
// suspend-time hint), giving up after kWaitLimitPoll polls.
#ifndef SOL_GEMM_PAIR_POLL
#define SOL_GEMM_PAIR_POLL 1
#endif
constexpr uint32_t kWaitLimitPoll = 1u << 26;

template <bool PAIR> __device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, Bars* b)
{
    const uint32_t limit = (PAIR && SOL_GEMM_PAIR_POLL) ? kWaitLimitPoll : kWaitLimit;
    for (uint32_t i = 0; i < limit; ++i) {
        bool ok;
        if (!PAIR)
            ok = mbar_try_wait(bar, parity);
        else if (SOL_GEMM_PAIR_POLL)
            ok = tc::mbar_poll_cluster(bar, parity);
        else
            ok = tc::mbar_try_wait_cluster(bar, parity, 1000000u);
        if (ok) return true;
        if ((i & 15u) == 15u && b->abort) return false;
    }
    return false;
}

__device__ __forceinline__ void raise_abort(Bars* b, uint32_t code)
{
    b->abort = 1;
    atomicOr(&g_gemm_error, code);
}

// ---------------------------------------------------------------------------------
// Producer (one thread per CTA): for every (tile, k-block) wait until the stage slot is
// free, then copy this CTA's 128 rows of A and its rows of B into it.  B rows of a tile:
// [n0, n0+128) and [n1, n1+128), with n0 = 128*n_blk (gated half) and n1 = inner +
// 128*n_blk (multiplying half) for SwiGLU, else n0 = 256*n_blk and n1 = n0 + 128; a single
// CTA loads both, CTA r of a pair loads n_r.  Rows of A past M read as zeros (tensor-map
// bounds).  The copies complete on this CTA's full[s], except those of a pair's peer
// without the transform, which complete on the leader's full[s]: the leader arms it for
// the bytes of both CTAs (the peer's copies may land before the leader arms the phase;
// the phase cannot complete before the leader's arrival), so the peer makes no remote
// arrival, whose cluster-scope release would cost more than the copy issue itself.
template <int EPI, bool PRO, bool FOLD, bool PAIR>
__device__ void run_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const Params& p, uint8_t* ring,
                             Bars* b, const Where& w)
{
    using S = Shape<PAIR>;
    const bool remote = PAIR && !PRO && w.rank == 1;  // this CTA's copies complete on the leader
    const int kblocks = p.K / BK;
    int s = 0;
    uint32_t phase = 0;
    int32_t last_parity[MAX_STAGES];
#pragma unroll
    for (int i = 0; i < MAX_STAGES; ++i) last_parity[i] = -1;

    Pass q = pass_begin();
    while (!b->abort && next_pass<PAIR, FOLD>(q, p, w)) {
        const int64_t m_blk = q.m_blk;
        const int32_t n_blk = q.n_blk;
        const int32_t y_a = (int32_t)(m_blk * S::TILE_M + (int64_t)w.rank * BM);
        // with the fold, B is this pass's modulation row's block of folded weights
        const int32_t nr = FOLD ? q.r * p.n_w : 0;
        const int32_t n0 = nr + (EPI == EPI_SWIGLU ? n_blk * (BN / 2) : n_blk * BN);
        const int32_t n1 = EPI == EPI_SWIGLU ? nr + p.inner + n_blk * (BN / 2) : n0 + BN / 2;
        for (int kb = 0; kb < kblocks; ++kb) {
            if (!wait_or_abort<PAIR>(smem_u32(&b->empty[s]), phase ^ 1u, b)) {
                raise_abort(b, 1u);
                break;
            }
            const uint32_t dst = smem_u32(ring + (size_t)s * S::STAGE_BYTES);
            if (remote) {
                // no arrival from the peer: the leader armed full[s] for both CTAs' bytes
                const uint32_t bar = tc::mapa(smem_u32(&b->full[s]), 0);
                tc::tma_load_2d_pair(dst, tmA, kb * BK, y_a, bar);
                tc::tma_load_2d_pair(dst + A_BYTES, tmB, kb * BK, n1, bar);
            } else {
                const uint32_t full = smem_u32(&b->full[s]);
                mbar_arrive_expect_tx(full, (PAIR && !PRO) ? 2 * S::STAGE_BYTES : S::STAGE_BYTES);
                tc::tma_load_2d(dst, tmA, kb * BK, y_a, full);
                if (PAIR) {
                    tc::tma_load_2d(dst + A_BYTES, tmB, kb * BK, w.rank == 0 ? n0 : n1, full);
                } else {
                    tc::tma_load_2d(dst + A_BYTES, tmB, kb * BK, n0, full);
                    tc::tma_load_2d(dst + A_BYTES + S::B_BYTES / 2, tmB, kb * BK, n1, full);
                }
            }
            last_parity[s] = (int32_t)phase;
            if (++s == S::STAGES) {
                s = 0;
                phase ^= 1u;
            }
        }
    }
    // Teardown: every copy issued must have landed before the CTA may exit.  A peer whose
    // copies complete on the leader hands its last phase per stage to the leader, which
    // waits for them between two cluster barriers at the end of the kernel.
    if (remote) {
#pragma unroll
        for (int i = 0; i < MAX_STAGES; ++i)
            tc::st_cluster_u32(tc::mapa(smem_u32(&b->peer_last[i]), 0), (uint32_t)last_parity[i]);
        return;
    }
#pragma unroll
    for (int i = 0; i < MAX_STAGES; ++i)
        if (last_parity[i] >= 0 && !mbar_wait_bounded(smem_u32(&b->full[i]), (uint32_t)last_parity[i], kWaitLimit))
            atomicOr(&g_gemm_error, 2u);
}

// ---------------------------------------------------------------------------------
// MMA issuer: one thread (of the leader, in a pair).  Stage s is consumed once its copies
// landed (full[s], counting both CTAs' copies in a pair) or, with the AdaLN
// transform, once the transform warps (of both CTAs) rewrote it (ready[s]).  The slot is
// released by a commit to empty[s] of each CTA when the four MMAs reading it finish; a
// finished accumulator is announced by a commit to acc_full of each CTA.
template <bool PRO, bool FOLD, bool PAIR>
__device__ void run_mma(const Params& p, uint8_t* ring, Bars* b, const Where& w)
{
    using S = Shape<PAIR>;
    const int kblocks = p.K / BK;
    const uint32_t idesc = tc::idesc_bf16_f32(S::TILE_M, BN);
    int s = 0;
    uint32_t phase = 0;
    int64_t it = 0;
    Pass q = pass_begin();
    for (; !b->abort && next_pass<PAIR, FOLD>(q, p, w); ++it) {
        const int ab = (int)(it & 1);
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        if (!wait_or_abort<PAIR>(smem_u32(&b->acc_empty[ab]), acc_phase ^ 1u, b)) {
            raise_abort(b, 4u);
            break;
        }
        tc::fence_after_sync();
        const uint32_t d_tmem = b->tmem_base + (uint32_t)(ab * BN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
            bool got;
            if (PRO)
                got = wait_or_abort<PAIR>(smem_u32(&b->ready[s]), phase, b);
            else
                got = wait_or_abort<PAIR>(smem_u32(&b->full[s]), phase, b);
            if (!got) {
                raise_abort(b, 8u);
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const uint32_t a_addr = smem_u32(ring + (size_t)s * S::STAGE_BYTES);
            const uint64_t a_desc = tc::smem_desc_sw128(a_addr);
            const uint64_t b_desc = tc::smem_desc_sw128(a_addr + A_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk) {
                // advance K by 16 elements = 32 bytes inside the swizzle row (field >> 4)
                const uint64_t da = a_desc + (uint64_t)(kk * 2), db = b_desc + (uint64_t)(kk * 2);
                const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
                if (PAIR)
                    tc::mma_bf16_pair(d_tmem, da, db, idesc, acc);
                else
                    tc::mma_bf16(d_tmem, da, db, idesc, acc);
            }
            const uint32_t e = smem_u32(&b->empty[s]);
            if (PAIR) {
                tc::commit_pair(e);
                tc::commit_pair(tc::mapa(e, 1));
            } else {
                tc::commit(e);
            }
            if (++s == S::STAGES) {
                s = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
        const uint32_t f = smem_u32(&b->acc_full[ab]);
        if (PAIR) {
            tc::commit_pair(f);
            tc::commit_pair(tc::mapa(f, 1));
        } else {
            tc::commit(f);
        }
    }
    // Teardown: wait for every MMA this thread issued.
    if (PAIR)
        tc::commit_pair(smem_u32(&b->drain));
    else
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

// AdaLN folded into the weights: the accumulator row holds x . V_r^T; the projection of
// h = (x - mean) * rstd * (1 + scale_r) + shift_r is rstd * (acc - mean * c_r) + b_r.
struct FoldRow {
    float mu, rs;
    const float* c;  // c_r + the tile's first column
    const float* b;  // b_r + the tile's first column
};

template <bool FOLD> __device__ __forceinline__ void fold32(float* v, const FoldRow& f, int col)
{
    if constexpr (FOLD) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 c4 = __ldg(reinterpret_cast<const float4*>(f.c + col) + j);
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(f.b + col) + j);
            v[4 * j + 0] = fmaf(f.rs, fmaf(-f.mu, c4.x, v[4 * j + 0]), b4.x);
            v[4 * j + 1] = fmaf(f.rs, fmaf(-f.mu, c4.y, v[4 * j + 1]), b4.y);
            v[4 * j + 2] = fmaf(f.rs, fmaf(-f.mu, c4.z, v[4 * j + 2]), b4.z);
            v[4 * j + 3] = fmaf(f.rs, fmaf(-f.mu, c4.w, v[4 * j + 3]), b4.w);
        }
    }
}

// One 128-wide head vector of the accumulator row (TMEM columns taddr .. +127):
// v / sqrt(mean(v^2) + eps) * w, then the interleaved 3D rotation, stored to dst.  The
// vector is read from TMEM once and held in registers (a second read would compete with
// the MMAs writing the other accumulator).
template <bool FOLD>
__device__ __forceinline__ void qk_head(uint32_t taddr, bool live, const bf16* w, const Params& p, int p0, int p1,
                                        int p2, bf16* dst, const FoldRow& fr, int col)
{
    // the whole head vector in registers: one read of its 128 TMEM columns
    float v[128];
#pragma unroll
    for (int c = 0; c < 4; ++c) tc::ld32(taddr + 32 * c, v + 32 * c);
    if (!live) return;
#pragma unroll
    for (int c = 0; c < 4; ++c) fold32<FOLD>(v + 32 * c, fr, col + 32 * c);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 128; ++i) ss = fmaf(v[i], v[i], ss);
    const float r = rsqrtf(ss * (1.f / 128.f) + p.eps);
    const int h0 = p.rope.half[0], h01 = p.rope.half[0] + p.rope.half[1];
#pragma unroll
    for (int c = 0; c < 16; ++c) {  // 8 elements (4 pairs) at a time
        float fw[8];
        if (w) {
            unpack<bf16>(ld_cached(w + 8 * c), fw);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) fw[e] = 1.f;
        }
        float o[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const int pi = 4 * c + m;  // pair index inside the head
            const float2* tab;
            if (pi < h0)
                tab = p.rope.tab[0] + pi + (int64_t)p0 * p.rope.half[0];
            else if (pi < h01)
                tab = p.rope.tab[1] + (pi - h0) + (int64_t)p1 * p.rope.half[1];
            else
                tab = p.rope.tab[2] + (pi - h01) + (int64_t)p2 * p.rope.half[2];
            const float2 cs = __ldg(tab);
            const float a = v[8 * c + 2 * m] * r * fw[2 * m];
            const float b = v[8 * c + 2 * m + 1] * r * fw[2 * m + 1];
            o[2 * m] = a * cs.x - b * cs.y;
            o[2 * m + 1] = a * cs.y + b * cs.x;
        }
        *reinterpret_cast<uint4*>(dst + 8 * c) = pack<bf16>(o);
    }
}

// Epilogue warps 2 .. 2+EW-1: thread (warp w, lane l) owns accumulator row 32*(w % 4) + l
// of this CTA's 128 rows (the TMEM lane quarter warp w may access) and, with EW = 8, half
// of its 256 columns ((w - 2) / 4 picks the half; a half is one head of the QKV epilogue).
// A drained accumulator is announced to the leader's acc_empty (one arrival per warp of
// each CTA).
template <int EPI, bool FOLD, bool PAIR, int EW>
__device__ void run_epilogue(const Params& p, Bars* b, const Where& w)
{
    constexpr int H = EW / 4;  // column parts per accumulator row
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    const int part = (warp - EPI_WARP0) / 4;  // this thread's part of the 256 columns
    int64_t it = 0;
    Pass q = pass_begin();
    for (; next_pass<PAIR, FOLD>(q, p, w); ++it) {
        const int ab = (int)(it & 1);
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        const bool got = wait_or_abort<PAIR>(smem_u32(&b->acc_full[ab]), acc_phase, b);
        if (!__all_sync(0xffffffffu, got)) {
            raise_abort(b, 32u);
            break;
        }
        tc::fence_after_sync();
        const int64_t m_blk = q.m_blk;
        const int32_t n_blk = q.n_blk;
        const int64_t row = m_blk * Shape<PAIR>::TILE_M + (int64_t)w.rank * BM + quarter * 32 + lane;
        bool live = row < p.M;
        FoldRow fr{0.f, 0.f, nullptr, nullptr};
        if constexpr (FOLD) {
            // rows of another modulation row are stored by that row's pass
            if (live) live = mod_row(row, p.sel) == q.r;
            if (live) {
                const float2 st = __ldg(p.stats + row);
                fr.mu = st.x;
                fr.rs = st.y;
            }
            fr.c = p.fold_c + (int64_t)q.r * p.n_w;
            fr.b = p.fold_b + (int64_t)q.r * p.n_w;
        }
        const uint32_t tbase = b->tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(ab * BN);
        float v[32];

        if constexpr (EPI == EPI_STORE) {
            bf16* dst = p.out + row * p.ld_out + (int64_t)n_blk * BN;
#pragma unroll 1
            for (int c = part * (8 / H); c < (part + 1) * (8 / H); ++c) {
                tc::ld32(tbase + 32 * c, v);
                if (!live) continue;
                fold32<FOLD>(v, fr, n_blk * BN + 32 * c);
                store32(dst + 32 * c, v);
            }
        } else if constexpr (EPI == EPI_GATED) {
            const int64_t col0 = (int64_t)n_blk * BN;
            const bf16* xr = p.x + row * p.ld_x + col0;
            const bf16* gr = nullptr;
            if (live && p.gate) gr = p.gate + mod_row(row, p.sel) * p.ld_mod + col0;
            bf16* dst = p.out + row * p.ld_out + col0;
#pragma unroll 1
            for (int c = part * (8 / H); c < (part + 1) * (8 / H); ++c) {
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
            for (int c = part * (4 / H); c < (part + 1) * (4 / H); ++c) {
                tc::ld32(tbase + 32 * c, v);
                tc::ld32(tbase + BN / 2 + 32 * c, u);
                if (!live) continue;
                fold32<FOLD>(v, fr, n_blk * (BN / 2) + 32 * c);
                fold32<FOLD>(u, fr, p.inner + n_blk * (BN / 2) + 32 * c);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = silu_mul_fast(v[i], u[i]);
                store32(dst + 32 * c, v);
            }
        } else {  // EPI_QKROPE
            const int32_t col0 = n_blk * BN;
            bf16* dst = p.out + row * p.ld_out + col0;
            if (col0 >= p.qk_cols) {  // v heads: as projected
#pragma unroll 1
                for (int c = part * (8 / H); c < (part + 1) * (8 / H); ++c) {
                    tc::ld32(tbase + 32 * c, v);
                    if (!live) continue;
                    fold32<FOLD>(v, fr, col0 + 32 * c);
                    store32(dst + 32 * c, v);
                }
            } else {
                int p0 = 0, p1 = 0, p2 = 0;
                if (live) token_pos(row, p, p0, p1, p2);
                const bf16* w = col0 < p.qk_cols / 2 ? p.wq : p.wk;
#pragma unroll 1
                for (int hh = part * (2 / H); hh < (part + 1) * (2 / H); ++hh)
                    qk_head<FOLD>(tbase + 128 * hh, live, w, p, p0, p1, p2, dst + 128 * hh, fr, col0 + 128 * hh);
            }
        }
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) {
            // the leader's acc_empty (this CTA's own when single)
            const uint32_t e = smem_u32(&b->acc_empty[ab]);
            if (PAIR)
                tc::mbar_arrive_cluster(tc::mapa(e, 0));
            else
                tc::mbar_arrive(e);
        }
    }
}


// ---------------------------------------------------------------------------------
// AdaLN operand transform (warps 6 and up: XFORM_GROUPS groups of four warps taking
// alternate k-blocks, so a group has XFORM_GROUPS MMA stage times per k-block).  The
// tensor copy lands the x tile (bf16, 128-byte swizzle) in the stage's A slot; the group
// rewrites it in place as
//     h = fma(fma(x, rstd, -mean * rstd), 1 + scale, shift)       (fp32, stored bf16)
// and arrives on the leader's ready[s], which the MMA waits for instead of full[s] (the
// transform itself waits for this CTA's full[s]).
// Mapping: lane L of warp w (of the group) handles row m = 4w + L/8 + 16j, j = 0..7, and
// logical 16-byte chunk kc = (L % 8) ^ (4 * (L / 16)) of each row (columns 8*kc ..
// 8*kc+7 of the k-block).  Logical chunk kc of row m sits at physical chunk kc ^ (m % 8),
// which is the same for all j (16j = 0 mod 8), so a thread's chunk position is fixed.
// The eight lanes of a quarter-warp (L/8 fixed) hit eight different chunks, and so do
// lanes {0-3, 16-19} (and the other such pairs: their chunk sets differ by the xor with
// 4 ^ 2), so a 128-bit shared access is conflict-free under either lane grouping.  When
// its rows share one modulation row (a tile inside one sample and one stream) the thread
// holds that row's 1 + scale and shift for its eight columns, fetched one k-block ahead;
// otherwise each row loads its own.  Rows past M stay zero (never stored).  Each thread
// fences its generic-proxy stores before its warp arrives, so the tensor core (async
// proxy) reads the rewritten tile.
#ifndef SOL_GEMM_XFORM_GROUPS
#define SOL_GEMM_XFORM_GROUPS 2
#endif
constexpr int XFORM_GROUPS = SOL_GEMM_XFORM_GROUPS;
constexpr int XFORM_WARPS = 4;
constexpr int XFORM_THREADS = 32 * XFORM_WARPS * XFORM_GROUPS;
// every stage must always belong to the same group (XFORM_WARPS arrivals per CTA and use)
static_assert(Shape<false>::STAGES % XFORM_GROUPS == 0, "the transform groups must divide the stage count");
// pairs take the transform only when the groups divide their ring too
constexpr bool kPairTransform = Shape<true>::STAGES % XFORM_GROUPS == 0;

__device__ __forceinline__ uint4 lds128(uint32_t a)
{
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void sts128(uint32_t a, const uint4& v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void load_mod8(const Params& p, int64_t r, int k0, float2* g, float2* sh)
{
    if (p.scale) {
        unpack2<bf16>(ld_cached(p.scale + r * p.ld_mod + k0), g);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) g[e] = make_float2(0.f, 0.f);
    }
    if (p.shift) {
        unpack2<bf16>(ld_cached(p.shift + r * p.ld_mod + k0), sh);
    } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) sh[e] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) g[e] = __fadd2_rn(make_float2(1.f, 1.f), g[e]);
}

template <bool PAIR>
__device__ void run_transform(const Params& p, uint8_t* ring, Bars* b, const Where& w)
{
    using S = Shape<PAIR>;
    const int tg = threadIdx.x - XFORM_WARP0 * 32;
    const int lane = threadIdx.x & 31;
    const int group = tg / (32 * XFORM_WARPS);
    const int wg = (tg % (32 * XFORM_WARPS)) >> 5;  // warp within the group
    const int r8 = 4 * wg + (lane >> 3);            // first row, 0..15
    const int kc = (lane & 7) ^ (4 * (lane >> 4));
    const int phys = kc ^ (r8 & 7);
    const int kblocks = p.K / BK;
    const uint32_t ring_s = smem_u32(ring);
    int64_t kglob = 0;                              // k-blocks of earlier tiles: ring position
    for (int64_t tile = w.worker; tile < p.num_tiles; tile += w.n_workers) {
        int64_t m_blk;
        int32_t n_blk;
        tile_coords<PAIR>(tile, p, m_blk, n_blk);
        const int64_t row0 = m_blk * S::TILE_M + (int64_t)w.rank * BM + r8;
        float2 ac[8];                                // (rstd, -mean * rstd) per row
        uint32_t live = 0;
        bool uniform = true;
        int64_t rmod0 = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int64_t row = row0 + 16 * j;
            ac[j] = make_float2(0.f, 0.f);
            if (row < p.M) {
                const float2 st = __ldg(p.stats + row);
                ac[j] = make_float2(st.y, -st.x * st.y);
                const int64_t r = mod_row(row, p.sel);
                if (j == 0) rmod0 = r;
                else if (r != rmod0) uniform = false;
                live |= 1u << j;
            }
        }
        int kb = (int)(((group - kglob % XFORM_GROUPS) % XFORM_GROUPS + XFORM_GROUPS) % XFORM_GROUPS);
        float2 g[4], sh[4], gn[4], shn[4];
        if (uniform && kb < kblocks) load_mod8(p, rmod0, kb * BK + 8 * kc, g, sh);
        bool ok = true;
        for (; kb < kblocks; kb += XFORM_GROUPS) {
            const int64_t kg = kglob + kb;
            const int s = (int)(kg % S::STAGES);
            const uint32_t phase = (uint32_t)((kg / S::STAGES) & 1);
            const int k0 = kb * BK + 8 * kc;
            if (uniform && kb + XFORM_GROUPS < kblocks) load_mod8(p, rmod0, k0 + XFORM_GROUPS * BK, gn, shn);
            if (!wait_or_abort<PAIR>(smem_u32(&b->full[s]), phase, b)) {
                raise_abort(b, 64u);
                ok = false;
                break;
            }
            const uint32_t base = ring_s + (uint32_t)(s * S::STAGE_BYTES + 16 * phys + r8 * 128);
            uint4 cell[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                if (live >> j & 1u) cell[j] = lds128(base + 16 * 128 * j);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (!(live >> j & 1u)) continue;
                if (!uniform) load_mod8(p, mod_row(row0 + 16 * j, p.sel), k0, g, sh);
                float2 f[4], h[4];
                unpack2<bf16>(cell[j], f);
                const float2 a2 = make_float2(ac[j].x, ac[j].x), c2 = make_float2(ac[j].y, ac[j].y);
#pragma unroll
                for (int e = 0; e < 4; ++e) h[e] = __ffma2_rn(__ffma2_rn(f[e], a2, c2), g[e], sh[e]);
                sts128(base + 16 * 128 * j, pack2<bf16>(h));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                // the leader's ready[s] (this CTA's own when single)
                const uint32_t r = smem_u32(&b->ready[s]);
                if (PAIR)
                    tc::mbar_arrive_cluster(tc::mapa(r, 0));
                else
                    tc::mbar_arrive(r);
            }
            if (uniform) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    g[e] = gn[e];
                    sh[e] = shn[e];
                }
            }
        }
        if (!ok) break;
        kglob += kblocks;
    }
}


// ---------------------------------------------------------------------------------
// The kernel: roles by warp (see the file header).
template <int EPI, bool PRO> __host__ __device__ constexpr int block_threads()
{
    return PRO ? 192 + XFORM_THREADS : 64 + 32 * epi_warps<EPI, false>();
}

template <int EPI, bool PRO, bool FOLD, bool PAIR>
__global__ void __launch_bounds__(block_threads<EPI, PRO>(), 1)
    k_linear(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ Params p)
{
    using S = Shape<PAIR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    Bars* b = reinterpret_cast<Bars*>(ring + (size_t)S::STAGES * S::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Where w = where<PAIR>();

    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < S::STAGES; ++i) {
            mbar_init(smem_u32(&b->full[i]), 1);
            mbar_init(smem_u32(&b->ready[i]), (PAIR ? 2 : 1) * XFORM_WARPS);  // one per warp of each CTA
            mbar_init(smem_u32(&b->empty[i]), 1);
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&b->acc_full[i]), 1);
            mbar_init(smem_u32(&b->acc_empty[i]), (PAIR ? 2 : 1) * epi_warps<EPI, PRO>());  // per epilogue warp, each CTA
        }
        mbar_init(smem_u32(&b->drain), 1);
#pragma unroll
        for (int i = 0; i < MAX_STAGES; ++i) b->peer_last[i] = -1;
        b->abort = 0;
        mbar_fence_init();
        tc::prefetch_tmap(&tmA);
        tc::prefetch_tmap(&tmB);
    }
    if (warp == MMA_WARP) {
        if constexpr (PAIR) {
            tc::tmem_alloc_pair(smem_u32(&b->tmem_base), TMEM_COLS);
            tc::tmem_relinquish_pair();
        } else {
            tc::tmem_alloc(smem_u32(&b->tmem_base), TMEM_COLS);
            tc::tmem_relinquish();
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if constexpr (PAIR) tc::cluster_sync();  // both CTAs' barriers exist before any remote arrival
    tc::fence_after_sync();

    if (warp == PRODUCER_WARP) {
        if (lane == 0) run_producer<EPI, PRO, FOLD, PAIR>(&tmA, &tmB, p, ring, b, w);
    } else if (warp == MMA_WARP) {
        if (lane == 0) {
            if (!PAIR || w.rank == 0) run_mma<PRO, FOLD, PAIR>(p, ring, b, w);
        }
    } else if (warp < EPI_WARP0 + epi_warps<EPI, PRO>()) {
        run_epilogue<EPI, FOLD, PAIR, epi_warps<EPI, PRO>()>(p, b, w);
    } else if (PRO) {
        run_transform<PAIR>(p, ring, b, w);
    }

    tc::fence_before_sync();
    __syncthreads();
    if constexpr (PAIR) {
        // the leader's MMAs into this CTA's TMEM have drained; the peer's last copy phases
        // are in the leader's peer_last
        tc::cluster_sync();
        if constexpr (!PRO) {
            if (w.rank == 0 && threadIdx.x == 0) {
#pragma unroll
                for (int i = 0; i < MAX_STAGES; ++i) {
                    const int32_t ph = b->peer_last[i];
                    if (ph >= 0 && !mbar_wait_bounded(smem_u32(&b->full[i]), (uint32_t)ph, kWaitLimit))
                        atomicOr(&g_gemm_error, 2u);
                }
            }
        }
        tc::cluster_sync();  // every copy into either CTA has landed
    }
    if (warp == MMA_WARP) {
        tc::fence_after_sync();
        if constexpr (PAIR)
            tc::tmem_dealloc_pair(b->tmem_base, TMEM_COLS);
        else
            tc::tmem_dealloc(b->tmem_base, TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------------
// Row statistics for the AdaLN variants: (mean, 1/sqrt(var + eps)) of each row of x,
// biased variance by two passes (the second re-reads the row from L1/L2).  One warp per
// row.  With rmask, also the set of modulation rows each 128-row block uses (bit r).
__global__ void __launch_bounds__(256) k_row_stats(float2* stats, uint32_t* rmask, ModSel sel, const bf16* x,
                                                   int64_t ld_x, int64_t M, int32_t d, float eps)
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
        if (lane == 0) {
            stats[row] = make_float2(mu, rsqrtf(var + eps));
            if (rmask) atomicOr(rmask + (row >> 7), 1u << (uint32_t)mod_row(row, sel));
        }
    }
}

// AdaLN folded into a linear layer's weights, per modulation row r and output column j:
//     V_r[j, k] = bf16(W[j, k] * (1 + scale_r[k]))       (the folded weights)
//     c_r[j]    = sum_k V_r[j, k]                         (fp32, of the rounded V)
//     b_r[j]    = sum_k shift_r[k] * W[j, k]              (fp32)
// so that LN-modulated rows project as rstd * (x . V_r^T - mean * c_r) + b_r.  One warp
// per (r, j); V is [R * n_w, K] with row stride K.
__global__ void __launch_bounds__(256) k_fold_weights(bf16* V, float* c, float* bsum, const bf16* W, int64_t ld_w,
                                                      int32_t n_w, int32_t K, const bf16* scale, const bf16* shift,
                                                      int64_t ld_mod, int32_t R)
{
    const int lane = threadIdx.x & 31;
    const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t wstep = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t total = (int64_t)R * n_w;
    for (int64_t idx = w0; idx < total; idx += wstep) {
        const int64_t r = idx / n_w, j = idx - r * n_w;
        const bf16* wr = W + j * ld_w;
        bf16* vr = V + idx * (int64_t)K;
        float cs = 0.f, bs = 0.f;
        for (int v = lane; v < K / 8; v += 32) {
            float fw[8], fg[8], fs[8];
            unpack<bf16>(ld_cached(wr + 8 * v), fw);
            if (scale) {
                unpack<bf16>(ld_cached(scale + r * ld_mod + 8 * v), fg);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) fg[e] = 0.f;
            }
            if (shift) {
                unpack<bf16>(ld_cached(shift + r * ld_mod + 8 * v), fs);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) fs[e] = 0.f;
            }
            float fv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                fv[e] = fw[e] * (1.f + fg[e]);
                bs = fmaf(fs[e], fw[e], bs);
            }
            const uint4 pv = pack<bf16>(fv);
            *reinterpret_cast<uint4*>(vr + 8 * v) = pv;
            float rv[8];
            unpack<bf16>(pv, rv);  // the rounded values the tensor cores will read
#pragma unroll
            for (int e = 0; e < 8; ++e) cs += rv[e];
        }
        cs = warp_sum(cs);
        bs = warp_sum(bs);
        if (lane == 0) {
            c[idx] = cs;
            bsum[idx] = bs;
        }
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
    const cuuint32_t box[2] = {(cuuint32_t)gemm::BK, (cuuint32_t)gemm::BM};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tile shape per variant, from the shape alone.  Measured on B200: CTA pairs are faster
// for the plain and epilogue-fused GEMMs (the copies per MMA drop by a third); with the
// AdaLN operand transform the single shape is faster (in a pair every transformed stage of
// the peer must be announced to the leader with a cluster-scope release, which costs more
// than the deeper ring saves).  A call of at most 128 rows also runs single: a pair's
// 256-row tile would leave the second CTA's half empty.
bool use_pair(bool transform, int64_t M) { return !transform && M > gemm::Shape<false>::TILE_M; }

template <int EPI, bool PRO, bool FOLD, bool PAIR>
cudaError_t launch_kernel(const CUtensorMap& ma, const CUtensorMap& mb, const gemm::Params& p, cudaStream_t s)
{
    auto kern = gemm::k_linear<EPI, PRO, FOLD, PAIR>;
    const size_t smem = gemm::smem_bytes<PAIR>();
    const int threads = gemm::block_threads<EPI, PRO>();
    // per device: the shared-memory attribute and the resident pair count
    constexpr int kMaxDevices = 64;
    static int attr_set[kMaxDevices] = {};
    static int max_pairs_dev[kMaxDevices] = {};
    static std::mutex mu;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::unique_lock<std::mutex> lk(mu);
    if (!attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_set[dev] = 1;
    }
    if constexpr (!PAIR) {
        lk.unlock();
        const int64_t grid = std::min<int64_t>(p.num_tiles, (int64_t)sm_count());
        kern<<<(unsigned)grid, threads, smem, s>>>(ma, mb, p);
        return cudaGetLastError();
    } else {
        cudaLaunchAttribute la[1];
        la[0].id = cudaLaunchAttributeClusterDimension;
        la[0].val.clusterDim.x = 2;
        la[0].val.clusterDim.y = 1;
        la[0].val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cfg.attrs = la;
        cfg.numAttrs = 1;
        // as many pairs as can be resident at once (persistent workers)
        if (!max_pairs_dev[dev]) {
            cudaLaunchConfig_t q = cfg;
            q.gridDim = dim3(2 * (sm_count() / 2));
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &q) != cudaSuccess || n < 1) n = sm_count() / 2;
            max_pairs_dev[dev] = n;
        }
        const int64_t pairs = std::min<int64_t>(p.num_tiles, (int64_t)max_pairs_dev[dev]);
        lk.unlock();
        cfg.gridDim = dim3((unsigned)(2 * pairs));
        return cudaLaunchKernelEx(&cfg, kern, ma, mb, p);
    }
}

template <int EPI, bool PRO, bool FOLD = false>
cudaError_t launch_shape(const CUtensorMap& ma, const CUtensorMap& mb, gemm::Params& p, int64_t M, cudaStream_t s)
{
    if constexpr (!PRO || gemm::kPairTransform) {
        if (use_pair(PRO, M)) {
            p.num_tiles = (M + gemm::Shape<true>::TILE_M - 1) / gemm::Shape<true>::TILE_M * (int64_t)p.n_tiles_n;
            return launch_kernel<EPI, PRO, FOLD, true>(ma, mb, p, s);
        }
    }
    p.num_tiles = (M + gemm::Shape<false>::TILE_M - 1) / gemm::Shape<false>::TILE_M * (int64_t)p.n_tiles_n;
    return launch_kernel<EPI, PRO, FOLD, false>(ma, mb, p, s);
}

// AdaLN strategy, chosen by the caller (sol_adaln_strategy):
//   stage (the fastest on B200): the AdaLN row kernel writes h (bf16) into the workspace
//     and the plain GEMM with the fused epilogue reads it -- one h round trip through
//     HBM, no change to the GEMM (AdaLN -> QKV + RoPE 4.17-4.23 ms vs 4.33-4.51 folded;
//     AdaLN -> up + SwiGLU 7.21-7.23 vs 7.63-7.92, at 32,768 tokens);
//   fold: the modulation folded into the weights, corrected in the epilogue (no h);
//   transform: the x tile rewritten as h in shared memory before the MMA (no h).

}  // namespace

size_t linear_smem_bytes() { return gemm::smem_bytes<true>(); }

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

    const int32_t strategy = adaln ? a.adaln_strategy : SOL_ADALN_TRANSFORM;
    if (adaln && strategy == SOL_ADALN_STAGE) {
        // h = AdaLN(x) into the workspace (K elements per row), then the GEMM on h
        const ModSel sel = a.sel ? *a.sel : ModSel{};
        cudaError_t e = launch_adaln_rows(SOL_DTYPE_BF16, nullptr, 0, a.fold_v, a.K, a.a, a.ld_a, nullptr, 0, nullptr,
                                          a.shift, a.scale, a.ld_mod, sel, a.M, a.K, a.eps, s);
        if (e != cudaSuccess) return e;
        if (!make_map(&ma, a.fold_v, (uint64_t)a.M, (uint64_t)a.K, (uint64_t)a.K)) {
            record_error("tensor map encoding failed for the staged AdaLN output");
            return cudaErrorInvalidValue;
        }
        adaln = false;
    }
    const bool fold = adaln && strategy == SOL_ADALN_FOLD;
    if (adaln) {
        const int64_t blocks = std::min<int64_t>((a.M + 7) / 8, (int64_t)sm_count() * 16);
        const ModSel sel = a.sel ? *a.sel : ModSel{};
        if (fold) {
            cudaError_t e = cudaMemsetAsync(a.rmask, 0, (size_t)((a.M + gemm::BM - 1) / gemm::BM) * 4, s);
            if (e != cudaSuccess) return e;
        }
        gemm::k_row_stats<<<(unsigned)blocks, 256, 0, s>>>(static_cast<float2*>(a.stats), fold ? a.rmask : nullptr,
                                                           sel, static_cast<const bf16*>(a.a), a.ld_a, a.M, a.K,
                                                           a.eps);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (fold) {
        // fold the modulation into the weights, then a plain GEMM on x with the correction
        // rstd * (acc - mean * c_r) + b_r in its epilogue
        const int64_t rows = (int64_t)a.n_mod_rows * a.N;
        const int64_t blocks = std::min<int64_t>((rows + 7) / 8, (int64_t)sm_count() * 16);
        gemm::k_fold_weights<<<(unsigned)blocks, 256, 0, s>>>(
            static_cast<bf16*>(a.fold_v), a.fold_c, a.fold_b, static_cast<const bf16*>(a.w), a.ld_w, a.N, a.K,
            static_cast<const bf16*>(a.scale), static_cast<const bf16*>(a.shift), a.ld_mod, a.n_mod_rows);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        if (!make_map(&mb, a.fold_v, (uint64_t)rows, (uint64_t)a.K, (uint64_t)a.K)) {
            record_error("tensor map encoding failed for the folded weights");
            return cudaErrorInvalidValue;
        }
        p.rmask = a.rmask;
        p.fold_c = a.fold_c;
        p.fold_b = a.fold_b;
        p.n_w = a.N;
        if (epi == LINEAR_STORE) return launch_shape<gemm::EPI_STORE, false, true>(ma, mb, p, a.M, s);
        if (epi == LINEAR_QKROPE) return launch_shape<gemm::EPI_QKROPE, false, true>(ma, mb, p, a.M, s);
        if (epi == LINEAR_SWIGLU) return launch_shape<gemm::EPI_SWIGLU, false, true>(ma, mb, p, a.M, s);
        return cudaErrorInvalidValue;
    }
    switch (epi) {
    case LINEAR_STORE:
        return adaln ? launch_shape<gemm::EPI_STORE, true>(ma, mb, p, a.M, s)
                     : launch_shape<gemm::EPI_STORE, false>(ma, mb, p, a.M, s);
    case LINEAR_GATED:
        return launch_shape<gemm::EPI_GATED, false>(ma, mb, p, a.M, s);
    case LINEAR_SWIGLU:
        return adaln ? launch_shape<gemm::EPI_SWIGLU, true>(ma, mb, p, a.M, s)
                     : launch_shape<gemm::EPI_SWIGLU, false>(ma, mb, p, a.M, s);
    case LINEAR_QKROPE:
        return adaln ? launch_shape<gemm::EPI_QKROPE, true>(ma, mb, p, a.M, s)
                     : launch_shape<gemm::EPI_QKROPE, false>(ma, mb, p, a.M, s);
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
