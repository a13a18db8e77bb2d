// k_rows.cu -- AdaLN modulation and the fused block prologue (gated residual -> AdaLN):
// the entry point launch_adaln_rows and the general kernels.  bf16 rows of the common
// widths go to the register-resident kernels of k_adaln_warp.cu (see the dispatch at the
// end of this file); fp32 and every other width take the kernels below.
//
// Bulk-copy ring kernel, k_adaln_bulk: a persistent CTA streams its rows (x, and y for the
// prologue) into a ring of `stages` shared-memory buffers with single-CTA 1-D bulk
// async copies completed on one mbarrier per buffer.  While a row is reduced, the next
// stages-1 rows of the CTA are already in flight, so HBM never waits on the reductions.
// A buffer is refilled as soon as every thread has copied its slice of the row into
// registers (right after the first reduction barrier).  Every mbarrier wait is bounded;
// on give-up the kernel records a device error flag, drains its own copies (bounded) and
// returns.
//
// Fallback kernel, k_adaln_rows (rows too wide for two shared-memory stages):
// one CTA per token row, rows walked with a grid stride.  The whole row lives in fp32
// registers (blockDim.x * U 16-byte vectors cover it), so x (and y) are read from HBM
// exactly once: the mean and then the variance are two reductions over registers
// (two-pass, so +-50 outliers and large offsets do not cancel), each a warp shuffle tree
// plus one shared-memory exchange.  The residual sum x' = x + gate*y stays unrounded in
// registers for the norm; only its stored copy is rounded.  Modulation rows come
// through the read-only path and stay L1/L2 resident across rows of the same sample.
#include <atomic>

#include "common.cuh"
#include "launch.h"

#ifndef SOL_ADALN_FOUR_WARPS
#define SOL_ADALN_FOUR_WARPS 1  // plain AdaLN on the four-warp prologue kernel (no residual); 0: one warp per row
#endif

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

// Bit 0: a bulk-copy wait in this file's kernels gave up.  Read by sol_device_errors().
static __device__ unsigned int g_rows_error;

// Launch policy of the bulk kernel per op (measured on B200 at d = 5120): AdaLN keeps
// its modulation rows as stored (bf16) so that five CTAs fit an SM; the prologue widens
// shift and 1+scale to fp32 once per row change and runs two CTAs with a two-deep ring.
#ifndef SOL_ROWS_UPREF_FIRST
#define SOL_ROWS_UPREF_FIRST 4  // first choice of 16-byte vectors per thread
#endif
#ifndef SOL_ROWS_ADALN_MOD_F32
#define SOL_ROWS_ADALN_MOD_F32 0
#endif
#ifndef SOL_ROWS_ADALN_MAX_CTAS
#define SOL_ROWS_ADALN_MAX_CTAS 5
#endif
#ifndef SOL_ROWS_ADALN_MAX_STAGES
#define SOL_ROWS_ADALN_MAX_STAGES 6
#endif
#ifndef SOL_ROWS_PRO_MOD_F32
#define SOL_ROWS_PRO_MOD_F32 1
#endif
#ifndef SOL_ROWS_PRO_MAX_CTAS
#define SOL_ROWS_PRO_MAX_CTAS 2
#endif
#ifndef SOL_ROWS_PRO_MAX_STAGES
#define SOL_ROWS_PRO_MAX_STAGES 2
#endif

constexpr uint32_t kWaitLimit = 4096;  // polls of <= ~1 ms each: a few seconds at most
constexpr int kMaxStages = 8;

template <typename T, int U, bool RESID, bool MODF32>
__global__ void __launch_bounds__(512)
k_adaln_bulk(T* x_out, int64_t ld_xo, T* h, int64_t ld_h, const T* x, int64_t ld_x,
             const T* __restrict__ y, int64_t ld_y, const T* __restrict__ gate,
             const T* __restrict__ shift, const T* __restrict__ scale, int64_t ld_mod, ModSel sel,
             int64_t n_tokens, int32_t vpr, int32_t stages, float inv_d, float eps)
{
    constexpr int E = Vec<T>::N;   // elements per 16-byte vector
    constexpr int P = E / 2;       // fp32 pairs per vector
    constexpr int NIN = RESID ? 2 : 1;
    extern __shared__ __align__(128) uint8_t smem_dyn[];
    __shared__ __align__(8) uint64_t bars[kMaxStages];
    __shared__ float4 red[2][16];  // per warp (n, mean, M2, sum), two rows deep
    const uint32_t row_bytes = (uint32_t)vpr * 16u;
    const int d = vpr * E;
    const int64_t step = gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;

    // layout: [1 + scale][shift][gate (T, d) if RESID][ring]; scale and shift are fp32
    // (d floats each) when MODF32, else rows as stored (T)
    constexpr size_t kModElem = MODF32 ? sizeof(float) : sizeof(T);
    float* scale1_s = reinterpret_cast<float*>(smem_dyn);
    float* shift_s = reinterpret_cast<float*>(smem_dyn + (size_t)d * kModElem);
    uint4* gate_s = reinterpret_cast<uint4*>(smem_dyn + 2 * (size_t)d * kModElem);
    uint8_t* ring0 = smem_dyn + 2 * (size_t)d * kModElem + (RESID ? row_bytes : 0u);
    auto ring = [&](int s, int i) { return ring0 + (size_t)(s * NIN + i) * row_bytes; };
    auto issue = [&](int s, int64_t row) {
        const uint32_t bar = smem_u32(&bars[s]);
        mbar_arrive_expect_tx(bar, NIN * row_bytes);
        bulk_g2s(smem_u32(ring(s, 0)), x + row * ld_x, row_bytes, bar);
        if constexpr (RESID) bulk_g2s(smem_u32(ring(s, 1)), y + row * ld_y, row_bytes, bar);
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(smem_u32(&bars[s]), 1);
        mbar_fence_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            const int64_t row = blockIdx.x + (int64_t)s * step;
            if (row < n_tokens) issue(s, row);
        }
    }

    // valid elements of this warp: columns warp*32 + lane + u*blockDim.x below vpr
    float wcnt = 0.f;
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c0 = u * (int)blockDim.x + warp * 32;
        wcnt += (float)(E * max(0, min(32, vpr - c0)));
    }
    const float inv_wcnt = 1.f / wcnt;
    const bool full = (int)blockDim.x * U == vpr;  // no idle lanes: equal counts everywhere

    int k = 0, s = 0;
    uint32_t parity = 0;
    int64_t cur_mr = -1;
    for (int64_t row = blockIdx.x; row < n_tokens; row += step, ++k) {
        // modulation rows of this row, widened once per change (CTA-uniform branch)
        const int64_t mr = mod_row(row, sel);
        if (mr != cur_mr) {
            __syncthreads();  // nobody still reads the previous ones
            for (int c = threadIdx.x; c < vpr; c += blockDim.x) {
                const int64_t off = mr * ld_mod + (int64_t)c * E;
                if constexpr (MODF32) {
                float2 f[P];
                unpack2<T>(scale ? ld_cached(scale + off) : make_uint4(0u, 0u, 0u, 0u), f);
#pragma unroll
                for (int i = 0; i < P; ++i)
                    reinterpret_cast<float2*>(scale1_s)[c * P + i] = __fadd2_rn(f[i], make_float2(1.f, 1.f));
                unpack2<T>(shift ? ld_cached(shift + off) : make_uint4(0u, 0u, 0u, 0u), f);
#pragma unroll
                for (int i = 0; i < P; ++i) reinterpret_cast<float2*>(shift_s)[c * P + i] = f[i];
                } else {
                reinterpret_cast<uint4*>(scale1_s)[c] = scale ? ld_cached(scale + off) : make_uint4(0u, 0u, 0u, 0u);
                reinterpret_cast<uint4*>(shift_s)[c] = shift ? ld_cached(shift + off) : make_uint4(0u, 0u, 0u, 0u);
                }
                if constexpr (RESID) gate_s[c] = gate ? ld_cached(gate + off) : make_uint4(0u, 0u, 0u, 0u);
            }
            __syncthreads();
            cur_mr = mr;
        }
        const bool ok = mbar_wait_bounded(smem_u32(&bars[s]), parity, kWaitLimit);

        // pass 1: x' = x (+ gate * y) into registers; one accumulator per vector (ILP)
        const uint4* xs = reinterpret_cast<const uint4*>(ring(s, 0));
        float2 v[U][P];
        float2 acc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int col = threadIdx.x + u * blockDim.x;
            acc[u] = make_float2(0.f, 0.f);
            if (col < vpr) {
                unpack2<T>(xs[col], v[u]);
                if constexpr (RESID) {
                    const uint4* ys = reinterpret_cast<const uint4*>(ring(s, 1));
                    float2 fy[P], fg[P];
                    unpack2<T>(ys[col], fy);
                    unpack2<T>(gate_s[col], fg);
#pragma unroll
                    for (int i = 0; i < P; ++i) v[u][i] = __ffma2_rn(fg[i], fy[i], v[u][i]);
                }
#pragma unroll
                for (int i = 0; i < P; ++i) acc[u] = __fadd2_rn(acc[u], v[u][i]);
            }
        }
#pragma unroll
        for (int u = 1; u < U; ++u) acc[0] = __fadd2_rn(acc[0], acc[u]);
        float wmean, wM2;
        if (full) {
            // every thread holds U*E elements: local two-pass mean and M2, then one
            // shuffle tree merging equal-count partials: mean = (ma + mb) / 2,
            // M2 = M2a + M2b + (mb - ma)^2 * n / 2 for n elements on each side
            const float lmean = (acc[0].x + acc[0].y) * (1.f / (U * E));
            const float2 lm2 = make_float2(-lmean, -lmean);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                acc[u] = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < P; ++i) {
                    const float2 c = __fadd2_rn(v[u][i], lm2);
                    acc[u] = __ffma2_rn(c, c, acc[u]);
                }
            }
#pragma unroll
            for (int u = 1; u < U; ++u) acc[0] = __fadd2_rn(acc[0], acc[u]);
            wmean = lmean;
            wM2 = acc[0].x + acc[0].y;
            float half_n = 0.5f * (U * E);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float mb = __shfl_xor_sync(0xffffffffu, wmean, off);
                const float m2b = __shfl_xor_sync(0xffffffffu, wM2, off);
                const float dm = mb - wmean;
                wM2 = fmaf(dm * dm, half_n, wM2 + m2b);
                wmean = 0.5f * (wmean + mb);
                half_n *= 2.f;
            }
        } else {
            // ragged row: warp sum, then M2 about the warp mean (two-pass inside the warp)
            const float wsum = warp_sum(acc[0].x + acc[0].y);
            wmean = wsum * inv_wcnt;
            const float2 wm2 = make_float2(-wmean, -wmean);
            float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int col = threadIdx.x + u * blockDim.x;
                if (col < vpr) {
#pragma unroll
                    for (int i = 0; i < P; ++i) {
                        const float2 c = __fadd2_rn(v[u][i], wm2);
                        a2 = __ffma2_rn(c, c, a2);
                    }
                }
            }
            wM2 = warp_sum(a2.x + a2.y);
        }
        if (lane == 0) red[k & 1][warp] = make_float4(wcnt, wmean, wM2, wcnt * wmean);
        // the one barrier of the row; it also votes on the bounded wait
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) {
                atomicOr(&g_rows_error, 1u);
                for (int j = 0; j < stages; ++j) {  // drain this CTA's copies in flight
                    const int kk = k + j;
                    if (row + (int64_t)j * step < n_tokens)
                        mbar_wait_bounded(smem_u32(&bars[kk % stages]), (uint32_t)(kk / stages) & 1u,
                                          kWaitLimit);
                }
            }
            return;
        }
        // every thread holds its slice of the row: refill this buffer `stages` rows ahead
        if (threadIdx.x == 0) {
            const int64_t nxt = row + (int64_t)stages * step;
            if (nxt < n_tokens) {
                fence_proxy_async_smem();
                issue(s, nxt);
            }
        }
        // row statistics: mean from the warp sums, M2 by the parallel-axis theorem
        // M2 = sum_w [M2_w + n_w (mean_w - mean)^2]  (exact, all terms >= 0)
        float tsum = 0.f;
        for (int i = 0; i < nw; ++i) tsum += red[k & 1][i].w;
        const float mean = tsum * inv_d;
        float m2 = 0.f;
        for (int i = 0; i < nw; ++i) {
            const float4 r = red[k & 1][i];
            const float dm = r.y - mean;
            m2 += fmaf(r.x * dm, dm, r.z);
        }
        const float rstd = rsqrtf(m2 * inv_d + eps);

        // output: h = (x' - mean) * rstd * (1 + scale) + shift
        const float2 nm2 = make_float2(-mean, -mean), r2 = make_float2(rstd, rstd);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int col = threadIdx.x + u * blockDim.x;
            if (col < vpr) {
                if constexpr (RESID) st_stream(x_out + row * ld_xo + (int64_t)col * E, pack2<T>(v[u]));
                float2 sc[P], sh[P];
                if constexpr (MODF32) {
#pragma unroll
                    for (int i = 0; i < P; ++i) {
                        sc[i] = reinterpret_cast<const float2*>(scale1_s)[col * P + i];
                        sh[i] = reinterpret_cast<const float2*>(shift_s)[col * P + i];
                    }
                } else {
                    unpack2<T>(reinterpret_cast<const uint4*>(scale1_s)[col], sc);
                    unpack2<T>(reinterpret_cast<const uint4*>(shift_s)[col], sh);
#pragma unroll
                    for (int i = 0; i < P; ++i) sc[i] = __fadd2_rn(sc[i], make_float2(1.f, 1.f));
                }
                float2 o[P];
#pragma unroll
                for (int i = 0; i < P; ++i) {
                    const float2 c = __fmul2_rn(__fadd2_rn(v[u][i], nm2), r2);
                    o[i] = __ffma2_rn(c, sc[i], sh[i]);
                }
                st_stream(h + row * ld_h + (int64_t)col * E, pack2<T>(o));
            }
        }
        if (++s == stages) {
            s = 0;
            parity ^= 1u;
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

namespace {

constexpr size_t kBulkSmemPerSM = 220 * 1024;  // dynamic shared memory we plan per SM
constexpr size_t kBulkSmemBudget = 200 * 1024;  // dynamic shared memory per CTA, at most

// Ring depth for `ctas` resident CTAs per SM: the shared memory left per CTA after the
// widened modulation rows, in stages of one (AdaLN) or two (prologue) rows; 0 if fewer
// than two stages fit.
int stages_for(int64_t vpr, int esize, bool resid, bool modf32, int max_stages, int ctas)
{
    const size_t row = (size_t)vpr * 16;
    const size_t d = row / (size_t)esize;
    const size_t stage = row * (resid ? 2 : 1);
    const size_t mod = 2 * d * (modf32 ? sizeof(float) : (size_t)esize) + (resid ? row : 0);
    size_t per_cta = kBulkSmemPerSM / (size_t)(ctas < 1 ? 1 : ctas);
    if (per_cta > kBulkSmemBudget) per_cta = kBulkSmemBudget;
    if (per_cta < mod + 2 * stage) return 0;
    size_t st = (per_cta - mod) / stage;
    if (st > (size_t)max_stages) st = max_stages;
    return (int)st;
}

size_t bulk_smem_bytes(int64_t vpr, int esize, bool resid, bool modf32, int stages)
{
    const size_t row = (size_t)vpr * 16;
    const size_t d = row / (size_t)esize;
    return 2 * d * (modf32 ? sizeof(float) : (size_t)esize) + (resid ? row : 0) +
           (size_t)stages * row * (resid ? 2 : 1);
}

// CTAs per SM the register file allows for `kfn` at `threads` threads (allocation in
// whole warps of 8-register granules), capped at `cap`.
int ctas_by_registers(const void* kfn, int threads, int cap)
{
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, kfn) != cudaSuccess || a.numRegs <= 0) return 1;
    const int regs = (a.numRegs + 7) / 8 * 8;
    const int warps = (threads + 31) / 32;
    int n = 65536 / (regs * 32 * warps);
    if (n > cap) n = cap;
    return n < 1 ? 1 : n;
}

// blockDim.x * U >= vpr, fewest idle lanes; U preference 4, 3, 6, 2, 8, 1: enough
// elements per thread to amortise the per-row work (index math, two reductions) that
// every thread repeats, without crowding the registers.
RowShape choose_bulk_shape(int64_t vpr)
{
    int kU[] = {4, 3, 6, 2, 8, 1};
    for (int i = 0; i < 6; ++i)  // move the configured first choice to the front
        if (kU[i] == SOL_ROWS_UPREF_FIRST) {
            for (int j = i; j > 0; --j) kU[j] = kU[j - 1];
            kU[0] = SOL_ROWS_UPREF_FIRST;
        }
    RowShape best{0, 0};
    int64_t best_waste = -1;
    for (int U : kU) {
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
cudaError_t run_bulk(void* x_out, int64_t ld_xo, void* h, int64_t ld_h, const void* x, int64_t ld_x,
                     const void* y, int64_t ld_y, const void* gate, const void* shift,
                     const void* scale, int64_t ld_mod, const ModSel& sel, int64_t n_tokens,
                     int64_t vpr, int threads, int64_t d, float eps, cudaStream_t s)
{
    constexpr bool MODF32 = RESID ? SOL_ROWS_PRO_MOD_F32 : SOL_ROWS_ADALN_MOD_F32;
    constexpr int kMaxCtas = RESID ? SOL_ROWS_PRO_MAX_CTAS : SOL_ROWS_ADALN_MAX_CTAS;
    constexpr int kMaxSt = RESID ? SOL_ROWS_PRO_MAX_STAGES : SOL_ROWS_ADALN_MAX_STAGES;
    const void* kfn = (const void*)k_adaln_bulk<T, U, RESID, MODF32>;
    // as many CTAs per SM as the registers allow (capped per op), then the deepest ring
    // (capped per op) that still fits them all
    int ctas = ctas_by_registers(kfn, threads, kMaxCtas);
    int stages = 0;
    for (; ctas >= 1 && (stages = stages_for(vpr, (int)sizeof(T), RESID, MODF32, kMaxSt, ctas)) == 0; --ctas) {
    }
    if (stages < 2) return cudaErrorInvalidConfiguration;
    const size_t smem = bulk_smem_bytes(vpr, (int)sizeof(T), RESID, MODF32, stages);
    static std::atomic<bool> attr_set[64];  // per instantiation and device; a repeated set is harmless
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kBulkSmemBudget);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kfn, cudaFuncAttributePreferredSharedMemoryCarveout,
                                     (int)cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    int64_t grid = (int64_t)ctas_per_sm(kfn, threads, smem) * sm_count();
    if (grid > n_tokens) grid = n_tokens;
    if (grid < 1) grid = 1;
    k_adaln_bulk<T, U, RESID, MODF32><<<(unsigned)grid, threads, smem, s>>>(
        (T*)x_out, ld_xo, (T*)h, ld_h, (const T*)x, ld_x, (const T*)y, ld_y, (const T*)gate,
        (const T*)shift, (const T*)scale, ld_mod, sel, n_tokens, (int32_t)vpr, stages,
        (float)(1.0 / (double)d), eps);
    return cudaGetLastError();
}

template <typename T, bool RESID>
cudaError_t dispatch_bulk(const RowShape& sh, void* x_out, int64_t ld_xo, void* h,
                          int64_t ld_h, const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                          const void* gate, const void* shift, const void* scale, int64_t ld_mod,
                          const ModSel& sel, int64_t n_tokens, int64_t vpr, int64_t d, float eps,
                          cudaStream_t s)
{
#define CASE(U)                                                                                    \
    case U:                                                                                        \
        return run_bulk<T, U, RESID>(x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate, shift, scale, \
                                     ld_mod, sel, n_tokens, vpr, sh.threads, d, eps, s);
    switch (sh.U) {
        CASE(1) CASE(2) CASE(3) CASE(4) CASE(6) CASE(8)
    default: return cudaErrorInvalidConfiguration;
    }
#undef CASE
}

}  // namespace

cudaError_t launch_adaln_rows(sol_dtype dt, void* x_out, int64_t ld_xo, void* h, int64_t ld_h,
                              const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                              const void* gate, const void* shift, const void* scale,
                              int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                              float eps, cudaStream_t s)
{
    if (!y && ld_x == ld_h && adaln_stage_fits(dt, d, n_tokens))
        return launch_adaln_stage(h, x, ld_h, shift, scale, ld_mod, sel, n_tokens, d, eps, s);
    if (!y && SOL_ADALN_FOUR_WARPS && ld_x == ld_h && prologue_regs_fits(dt, d))
        return launch_prologue_regs(nullptr, h, x, nullptr, nullptr, shift, scale, ld_h, ld_mod, sel, n_tokens, d,
                                    eps, s);
    if (!y && adaln_warp_fits(dt, d))
        return launch_adaln_warp(h, ld_h, x, ld_x, shift, scale, ld_mod, sel, n_tokens, d, eps, s);
    if (y && x_out && ld_xo == ld_h && ld_x == ld_h && ld_y == ld_h && prologue_regs_fits(dt, d))
        return launch_prologue_regs(x_out, h, x, y, gate, shift, scale, ld_h, ld_mod, sel, n_tokens, d, eps, s);
    const int64_t vpr = d / (dt == SOL_DTYPE_BF16 ? 8 : 4);
    const bool resid = y != nullptr;
    const bool bulk_fits =
        stages_for(vpr, dt == SOL_DTYPE_BF16 ? 2 : 4, resid,
                   resid ? SOL_ROWS_PRO_MOD_F32 : SOL_ROWS_ADALN_MOD_F32,
                   resid ? SOL_ROWS_PRO_MAX_STAGES : SOL_ROWS_ADALN_MAX_STAGES, 1) >= 2;
    const RowShape bsh = choose_bulk_shape(vpr);
    if (bulk_fits && bsh.threads > 0) {
        if (dt == SOL_DTYPE_BF16) {
            if (y)
                return dispatch_bulk<bf16, true>(bsh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y,
                                                 gate, shift, scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
            return dispatch_bulk<bf16, false>(bsh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate,
                                              shift, scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
        }
        if (y)
            return dispatch_bulk<float, true>(bsh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate,
                                              shift, scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
        return dispatch_bulk<float, false>(bsh, x_out, ld_xo, h, ld_h, x, ld_x, y, ld_y, gate,
                                           shift, scale, ld_mod, sel, n_tokens, vpr, d, eps, s);
    }
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

uint32_t rows_device_error(bool clear)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_rows_error, sizeof v) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_rows_error, &zero, sizeof zero);
    }
    return v;
}

}  // namespace sol
