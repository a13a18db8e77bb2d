// sol_block_host.cu -- sol_dit_block_host: one pass of the block's per-token hot path over
// host-resident tensors, with the host <-> device copies of each chunk overlapped with the
// compute of its neighbours [STM-RES, "SGLang acelera video do MiniMax-H3...", section
// "Resultado principal": the fused operators cut memory traffic and per-step launches;
// video and audio tokens share one packed DiT stack].
//
// Chunks never cross a sample, so each chunk is one call per operator with its sample's
// modulation rows (tokens_per_sample 0) and explicit positions: the host's positions, or,
// for the implicit row-major grid, positions generated on the device from the chunk's
// first token inside its sample.  Three streams and n_slots device buffers:
//   s_in    [wait: slot's previous chunk copied out] H2D copies of the chunk   -> in_done
//   s_comp  [wait: in_done] the five launches                                   -> comp_done
//   s_out   [wait: comp_done] D2H copies of the requested outputs               -> out_done
// One event per slot and stage suffices: each cudaStreamWaitEvent captures the event's
// latest record at the time it is enqueued, and the records of a slot follow each other in
// the order the waits need.
#include <cmath>
#include <cstdarg>
#include <cstdio>

#include "common.cuh"
#include "launch.h"
#include "sol.h"

namespace {

thread_local char g_msg[384];

sol_status fail(sol_status st, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    sol::record_error(g_msg);
    return st;
}

#define BH_CHECK(cond, st, ...)                    \
    do {                                           \
        if (!(cond)) return fail(st, __VA_ARGS__); \
    } while (0)

#define BH_CUDA(expr, what)                                                                    \
    do {                                                                                       \
        const cudaError_t e_ = (expr);                                                         \
        if (e_ != cudaSuccess) return fail(SOL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e_)); \
    } while (0)

#define BH_TRY(expr)                          \
    do {                                      \
        const sol_status st_ = (expr);        \
        if (st_ != SOL_OK) return st_;        \
    } while (0)

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t esize(sol_dtype dt) { return dt == SOL_DTYPE_BF16 ? 2 : 4; }

int64_t n_samples(const sol_block_host_desc& d)
{
    if (d.tokens_per_sample <= 0) return 1;
    return d.n_tokens > 0 ? (d.n_tokens + d.tokens_per_sample - 1) / d.tokens_per_sample : 1;
}

// Workspace: the per-call constants (six modulation tensors, wq, wk), then n_slots chunk
// buffers; every region 256-byte aligned.
struct Layout {
    size_t mod[6], wq, wk, consts;                        // offsets from the start
    size_t x, qkv, ya, u, ym, h1, x1, h2, act, x2, pos, sid, slot;  // offsets inside a slot
    int64_t chunk;                                       // tokens a slot holds
    size_t total;
};

Layout layout(const sol_block_host_desc& d, int64_t chunk_tokens, int32_t n_slots)
{
    Layout L{};
    const size_t e = esize(d.dt);
    const int64_t hd = (int64_t)d.n_heads * d.head_dim;
    size_t off = 0;
    const size_t mod_bytes = (size_t)(n_samples(d) * d.n_streams * d.d) * e;
    for (int i = 0; i < 6; ++i) {
        L.mod[i] = off;
        off = up256(off + mod_bytes);
    }
    L.wq = off;
    off = up256(off + (size_t)d.head_dim * e);
    L.wk = off;
    off = up256(off + (size_t)d.head_dim * e);
    L.consts = off;
    L.chunk = chunk_tokens < d.n_tokens ? chunk_tokens : (d.n_tokens > 0 ? d.n_tokens : 1);
    const size_t rows = (size_t)L.chunk;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = up256(o + bytes);
        return at;
    };
    L.x = take(rows * d.d * e);
    L.qkv = take(rows * 3 * hd * e);
    L.ya = take(rows * d.d * e);
    L.u = take(rows * 2 * d.inner * e);
    L.ym = take(rows * d.d * e);
    L.h1 = take(rows * d.d * e);
    L.x1 = take(rows * d.d * e);
    L.h2 = take(rows * d.d * e);
    L.act = take(rows * d.inner * e);
    L.x2 = take(rows * d.d * e);
    L.pos = take(rows * 3 * sizeof(int32_t));
    L.sid = take(rows);
    L.slot = o;
    L.total = L.consts + (size_t)n_slots * L.slot;
    return L;
}

bool sizes_ok(const sol_block_host_desc& d, int64_t chunk_tokens, int32_t n_slots)
{
    return (d.dt == SOL_DTYPE_F32 || d.dt == SOL_DTYPE_BF16) && d.n_tokens >= 0 && d.tokens_per_sample >= 0 &&
           d.n_streams >= 1 && d.n_streams <= 256 && d.d >= 8 && d.d <= (int64_t)1 << 20 && d.inner >= 8 &&
           d.inner <= (int64_t)1 << 22 && d.n_heads >= 1 && d.n_heads <= 4096 && d.head_dim >= 1 &&
           d.head_dim <= 4096 && chunk_tokens >= 1 && n_slots >= 1 && n_slots <= 64;
}

// Positions of `L` consecutive tokens of one sample whose first token is the sample's
// `first`-th, on the row-major grid_T x grid_H x grid_W grid.
__global__ void k_grid_positions(int32_t* pos, int64_t first, int64_t L, int32_t grid_H, int32_t grid_W)
{
    const int64_t hw = (int64_t)grid_H * grid_W;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t nl = first + i;
        pos[3 * i + 0] = (int32_t)(nl / hw);
        pos[3 * i + 1] = (int32_t)((nl / grid_W) % grid_H);
        pos[3 * i + 2] = (int32_t)(nl % grid_W);
    }
}

struct Events {
    cudaEvent_t ev[3 * 64 + 2] = {};
    int n = 0;
    ~Events()
    {
        for (int i = 0; i < n; ++i) cudaEventDestroy(ev[i]);  // released once they complete
    }
};

}  // namespace

extern "C" size_t sol_dit_block_host_workspace_bytes(const sol_block_host_desc* desc, int64_t chunk_tokens,
                                                     int32_t n_slots)
{
    if (!desc || !sizes_ok(*desc, chunk_tokens, n_slots)) return 0;
    return layout(*desc, chunk_tokens, n_slots).total;
}

extern "C" sol_status sol_dit_block_host(const sol_block_host_desc* desc, void* workspace, size_t workspace_bytes,
                                         int64_t chunk_tokens, int32_t n_slots, sol_stream_t s_in_,
                                         sol_stream_t s_comp_, sol_stream_t s_out_)
{
    BH_CHECK(desc, SOL_ERR_INVALID_ARGUMENT, "desc is NULL");
    const sol_block_host_desc& d = *desc;
    BH_CHECK(d.dt == SOL_DTYPE_F32 || d.dt == SOL_DTYPE_BF16, SOL_ERR_UNSUPPORTED, "dtype %d is not built",
             (int)d.dt);
    BH_CHECK(sizes_ok(d, chunk_tokens, n_slots), SOL_ERR_INVALID_ARGUMENT,
             "sizes out of range (n_tokens %lld, tokens_per_sample %lld, n_streams %d, d %lld, inner %lld, "
             "heads %d x %d, chunk_tokens %lld, n_slots %d)",
             (long long)d.n_tokens, (long long)d.tokens_per_sample, (int)d.n_streams, (long long)d.d,
             (long long)d.inner, (int)d.n_heads, (int)d.head_dim, (long long)chunk_tokens, (int)n_slots);
    const int e16 = d.dt == SOL_DTYPE_BF16 ? 8 : 4;
    BH_CHECK(d.d % e16 == 0 && d.inner % e16 == 0, SOL_ERR_MISALIGNED,
             "d (%lld) and inner (%lld) must be multiples of %d elements", (long long)d.d, (long long)d.inner, e16);
    BH_CHECK(std::isfinite(d.eps) && d.eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    BH_CHECK(d.rope, SOL_ERR_INVALID_ARGUMENT, "rope is NULL");
    if (!d.pos)
        BH_CHECK(d.grid_T >= 1 && d.grid_H >= 1 && d.grid_W >= 1 &&
                     (d.tokens_per_sample > 0 ? d.tokens_per_sample : d.n_tokens) <=
                         (int64_t)d.grid_T * d.grid_H * d.grid_W,
                 SOL_ERR_INVALID_ARGUMENT, "implicit positions need a grid_T x grid_H x grid_W grid holding a sample");
    BH_CHECK(s_in_ != s_comp_ && s_out_ != s_comp_ && s_in_ != s_out_, SOL_ERR_INVALID_ARGUMENT,
             "s_in, s_comp and s_out must be three distinct streams");
    if (d.n_tokens == 0) return SOL_OK;
    BH_CHECK(d.x && d.qkv && d.y_attn && d.u && d.y_mlp, SOL_ERR_INVALID_ARGUMENT,
             "x, qkv, y_attn, u and y_mlp are required");
    const Layout L = layout(d, chunk_tokens, n_slots);
    BH_CHECK(workspace, SOL_ERR_INVALID_ARGUMENT, "workspace is NULL");
    BH_CHECK((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, SOL_ERR_MISALIGNED,
             "workspace is not 256-byte aligned");
    BH_CHECK(workspace_bytes >= L.total, SOL_ERR_INVALID_ARGUMENT, "workspace of %zu bytes is below the %zu needed",
             workspace_bytes, L.total);

    // each operator checks its shape, dtype, eps and tables even on zero rows: one such call
    // per operator validates them before anything is enqueued (it launches nothing)
    {
        char* sb = static_cast<char*>(workspace) + L.consts;
        const int64_t hd3 = 3 * (int64_t)d.n_heads * d.head_dim;
        const sol_modsel sel0{nullptr, d.n_streams, 0};
        const int32_t* pos0 = reinterpret_cast<const int32_t*>(sb + L.pos);
        BH_TRY(sol_adaln_modulate(sb + L.h1, d.d, sb + L.x, d.d, nullptr, nullptr, d.d, sel0, 0, d.d, d.eps, d.dt,
                                  s_comp_));
        BH_TRY(sol_dit_epilogue(sb + L.qkv, hd3, nullptr, nullptr, pos0, d.grid_T, d.grid_H, d.grid_W, 0, d.rope, 0,
                                d.n_heads, d.head_dim, d.eps, d.dt, s_comp_));
        BH_TRY(sol_dit_prologue(sb + L.x1, sb + L.h2, sb + L.x, sb + L.ya, nullptr, nullptr, nullptr, d.d, d.d, sel0,
                                0, d.d, d.eps, d.dt, s_comp_));
        BH_TRY(sol_swiglu(sb + L.act, d.inner, sb + L.u, sb + L.u, 2 * d.inner, 0, d.inner, d.dt, s_comp_));
        BH_TRY(sol_gated_residual(sb + L.x2, d.d, sb + L.x1, d.d, sb + L.ym, d.d, nullptr, d.d, sel0, 0, d.d, d.dt,
                                  s_comp_));
    }

    const cudaStream_t s_in = (cudaStream_t)s_in_, s_comp = (cudaStream_t)s_comp_, s_out = (cudaStream_t)s_out_;
    char* ws = static_cast<char*>(workspace);
    const size_t e = esize(d.dt);
    const int64_t hd = (int64_t)d.n_heads * d.head_dim;
    const int64_t S = d.n_streams;
    const size_t mod_bytes = (size_t)(n_samples(d) * S * d.d) * e;

    Events ev;
    auto make = [&](cudaEvent_t* out) -> sol_status {
        BH_CUDA(cudaEventCreateWithFlags(out, cudaEventDisableTiming), "cudaEventCreateWithFlags");
        ++ev.n;
        return SOL_OK;
    };
    cudaEvent_t* start = &ev.ev[0];
    cudaEvent_t* done = &ev.ev[1];
    cudaEvent_t* in_done = &ev.ev[2];
    cudaEvent_t* comp_done = in_done + n_slots;
    cudaEvent_t* out_done = comp_done + n_slots;
    for (int i = 0; i < 2 + 3 * n_slots; ++i) BH_TRY(make(&ev.ev[i]));

    BH_CUDA(cudaEventRecord(*start, s_comp), "cudaEventRecord");
    BH_CUDA(cudaStreamWaitEvent(s_in, *start, 0), "cudaStreamWaitEvent");
    BH_CUDA(cudaStreamWaitEvent(s_out, *start, 0), "cudaStreamWaitEvent");

    // per-call constants: modulation rows and RMSNorm weights
    const void* mod_host[6] = {d.shift_msa, d.scale_msa, d.gate_msa, d.shift_mlp, d.scale_mlp, d.gate_mlp};
    const char* mod_dev[6];
    for (int i = 0; i < 6; ++i) {
        mod_dev[i] = nullptr;
        if (mod_host[i]) {
            BH_CUDA(cudaMemcpyAsync(ws + L.mod[i], mod_host[i], mod_bytes, cudaMemcpyHostToDevice, s_in),
                    "modulation rows H2D");
            mod_dev[i] = ws + L.mod[i];
        }
    }
    const void* wq_dev = nullptr;
    const void* wk_dev = nullptr;
    if (d.wq) {
        BH_CUDA(cudaMemcpyAsync(ws + L.wq, d.wq, (size_t)d.head_dim * e, cudaMemcpyHostToDevice, s_in), "wq H2D");
        wq_dev = ws + L.wq;
    }
    if (d.wk) {
        BH_CUDA(cudaMemcpyAsync(ws + L.wk, d.wk, (size_t)d.head_dim * e, cudaMemcpyHostToDevice, s_in), "wk H2D");
        wk_dev = ws + L.wk;
    }

    const int64_t tps = d.tokens_per_sample > 0 ? d.tokens_per_sample : d.n_tokens;
    const char* hx = static_cast<const char*>(d.x);
    const char* hqkv = static_cast<const char*>(d.qkv);
    const char* hya = static_cast<const char*>(d.y_attn);
    const char* hu = static_cast<const char*>(d.u);
    const char* hym = static_cast<const char*>(d.y_mlp);
    int64_t j = 0;
    for (int64_t b0 = 0; b0 < d.n_tokens; b0 += tps) {
        const int64_t b1 = b0 + tps < d.n_tokens ? b0 + tps : d.n_tokens;
        const int64_t b = b0 / tps;
        for (int64_t c0 = b0; c0 < b1; c0 += L.chunk, ++j) {
            const int64_t n = c0 + L.chunk < b1 ? L.chunk : b1 - c0;
            const int slot = (int)(j % n_slots);
            char* sb = ws + L.consts + (size_t)slot * L.slot;
            // ---- copy in (after the slot's previous chunk was copied out)
            if (j >= n_slots) BH_CUDA(cudaStreamWaitEvent(s_in, out_done[slot], 0), "cudaStreamWaitEvent");
            const size_t rd = (size_t)n * d.d * e;
            BH_CUDA(cudaMemcpyAsync(sb + L.x, hx + (size_t)c0 * d.d * e, rd, cudaMemcpyHostToDevice, s_in), "x H2D");
            BH_CUDA(cudaMemcpyAsync(sb + L.qkv, hqkv + (size_t)c0 * 3 * hd * e, (size_t)n * 3 * hd * e,
                                    cudaMemcpyHostToDevice, s_in), "qkv H2D");
            BH_CUDA(cudaMemcpyAsync(sb + L.ya, hya + (size_t)c0 * d.d * e, rd, cudaMemcpyHostToDevice, s_in),
                    "y_attn H2D");
            BH_CUDA(cudaMemcpyAsync(sb + L.u, hu + (size_t)c0 * 2 * d.inner * e, (size_t)n * 2 * d.inner * e,
                                    cudaMemcpyHostToDevice, s_in), "u H2D");
            BH_CUDA(cudaMemcpyAsync(sb + L.ym, hym + (size_t)c0 * d.d * e, rd, cudaMemcpyHostToDevice, s_in),
                    "y_mlp H2D");
            int32_t* pos_dev = reinterpret_cast<int32_t*>(sb + L.pos);
            if (d.pos) {
                BH_CUDA(cudaMemcpyAsync(pos_dev, d.pos + 3 * c0, (size_t)n * 3 * sizeof(int32_t),
                                        cudaMemcpyHostToDevice, s_in), "pos H2D");
            } else {
                const int64_t blocks = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
                k_grid_positions<<<(unsigned)blocks, 256, 0, s_in>>>(pos_dev, c0 - b0, n, d.grid_H, d.grid_W);
                BH_CUDA(cudaGetLastError(), "grid positions launch");
            }
            const uint8_t* sid_dev = nullptr;
            if (d.stream_id) {
                BH_CUDA(cudaMemcpyAsync(sb + L.sid, d.stream_id + c0, (size_t)n, cudaMemcpyHostToDevice, s_in),
                        "stream_id H2D");
                sid_dev = reinterpret_cast<const uint8_t*>(sb + L.sid);
            }
            BH_CUDA(cudaEventRecord(in_done[slot], s_in), "cudaEventRecord");

            // ---- compute
            BH_CUDA(cudaStreamWaitEvent(s_comp, in_done[slot], 0), "cudaStreamWaitEvent");
            const sol_modsel sel{sid_dev, (int32_t)S, 0};
            const int64_t mrow = b * S * d.d;  // this sample's rows of a modulation tensor
            auto mod = [&](int i) -> const void* { return mod_dev[i] ? mod_dev[i] + (size_t)mrow * e : nullptr; };
            BH_TRY(sol_adaln_modulate(sb + L.h1, d.d, sb + L.x, d.d, mod(0), mod(1), d.d, sel, n, d.d, d.eps, d.dt,
                                      s_comp_));
            BH_TRY(sol_dit_epilogue(sb + L.qkv, 3 * hd, wq_dev, wk_dev, pos_dev, d.grid_T, d.grid_H, d.grid_W, 0,
                                    d.rope, n, d.n_heads, d.head_dim, d.eps, d.dt, s_comp_));
            BH_TRY(sol_dit_prologue(sb + L.x1, sb + L.h2, sb + L.x, sb + L.ya, mod(2), mod(3), mod(4), d.d, d.d, sel,
                                    n, d.d, d.eps, d.dt, s_comp_));
            BH_TRY(sol_swiglu(sb + L.act, d.inner, sb + L.u, sb + L.u + (size_t)d.inner * e, 2 * d.inner, n, d.inner,
                              d.dt, s_comp_));
            BH_TRY(sol_gated_residual(sb + L.x2, d.d, sb + L.x1, d.d, sb + L.ym, d.d, mod(5), d.d, sel, n, d.d,
                                      d.dt, s_comp_));
            BH_CUDA(cudaEventRecord(comp_done[slot], s_comp), "cudaEventRecord");

            // ---- copy out
            BH_CUDA(cudaStreamWaitEvent(s_out, comp_done[slot], 0), "cudaStreamWaitEvent");
            struct Out {
                void* host;
                size_t off, width;
            } outs[5] = {{d.h1, L.h1, (size_t)d.d}, {d.x1, L.x1, (size_t)d.d}, {d.h2, L.h2, (size_t)d.d},
                         {d.act, L.act, (size_t)d.inner}, {d.x2, L.x2, (size_t)d.d}};
            for (const Out& o : outs)
                if (o.host)
                    BH_CUDA(cudaMemcpyAsync(static_cast<char*>(o.host) + (size_t)c0 * o.width * e, sb + o.off,
                                            (size_t)n * o.width * e, cudaMemcpyDeviceToHost, s_out), "output D2H");
            if (d.qk)
                BH_CUDA(cudaMemcpy2DAsync(static_cast<char*>(d.qk) + (size_t)c0 * 2 * hd * e, 2 * hd * e, sb + L.qkv,
                                          3 * hd * e, 2 * hd * e, (size_t)n, cudaMemcpyDeviceToHost, s_out),
                        "q|k D2H");
            BH_CUDA(cudaEventRecord(out_done[slot], s_out), "cudaEventRecord");
        }
    }
    BH_CUDA(cudaEventRecord(*done, s_out), "cudaEventRecord");
    BH_CUDA(cudaStreamWaitEvent(s_comp, *done, 0), "cudaStreamWaitEvent");
    return SOL_OK;
}
