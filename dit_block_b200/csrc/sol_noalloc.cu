// sol_noalloc.cu -- sol_qk_rmsnorm_rope3d_noalloc: QK RMSNorm + 3D RoPE for callers that
// must not allocate device memory.
//
// Who needs it: hosts that reserve device memory up front and forbid allocation while
// they run work -- inference engines whose memory pool already holds nearly all of HBM
// (a cudaMalloc there fails or fragments the pool), plugin interfaces whose execute
// callbacks must not allocate, and latency-critical loops where cudaMalloc's implicit
// device synchronisation is not acceptable.  The regular entry point needs a
// sol_rope3d handle, whose creation calls cudaMalloc; this variant does not.
//
// How: the cos/sin table lives in the file-scope device array below, of a fixed maximum
// size (kNoAllocRopeEntries float2 entries = 512 KiB, held by every GPU that loads this
// library until the process exits).  Each call rebuilds the part of the table it needs
// with a small kernel on the caller's stream, then runs the same QK kernel as
// sol_qk_rmsnorm_rope3d, in stream order.  Nothing in the table has to start at zero:
// every entry the QK kernel reads is written by the same call.  All calls share the
// one array, so two calls whose kernels overlap on the GPU (different streams, or
// different host threads without ordering) race on it.
//
// Set-up: the device address of the array is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on it; that
// first call should therefore come before any stream capture.  The address is kept for
// the life of the process, so it goes stale if the device's primary context is destroyed
// (cudaDeviceReset): the entry point is not for use after a reset.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "launch.h"
#include "sol.h"

namespace {

constexpr int64_t kNoAllocRopeEntries = SOL_NOALLOC_MAX_ROPE_ENTRIES;
static_assert(kNoAllocRopeEntries == 65536, "keep the header's stated maximum");

static __device__ __align__(256) float2 g_rope_noalloc_table[kNoAllocRopeEntries];

// One entry per (axis, position, pair): phi = p * theta^(-2j / dim_c), cos and sin
// evaluated in fp64 and rounded once to fp32 (the same rule as sol_rope3d_create).
__global__ void k_build_rope_table(float2* tab, int32_t half_t, int32_t half_h, int32_t half_w,
                                   int32_t max_t, int32_t max_h, int32_t max_w, double theta)
{
    const int64_t n_t = (int64_t)max_t * half_t;
    const int64_t n_h = (int64_t)max_h * half_h;
    const int64_t total = n_t + n_h + (int64_t)max_w * half_w;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        int64_t local = i;
        int32_t half = half_t;
        if (local >= n_t) {
            local -= n_t;
            half = half_h;
            if (local >= n_h) {
                local -= n_h;
                half = half_w;
            }
        }
        const int64_t p = local / half;
        const int32_t j = (int32_t)(local - p * half);
        const double phi = (double)p * pow(theta, -2.0 * (double)j / (double)(2 * half));
        double s, c;
        sincos(phi, &s, &c);
        tab[i] = make_float2((float)c, (float)s);
    }
}

std::mutex g_mu;
float2* g_table_ptr[64];  // device address of g_rope_noalloc_table, per device

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

#define NA_CHECK(cond, st, ...)                    \
    do {                                           \
        if (!(cond)) return fail(st, __VA_ARGS__); \
    } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

sol_status check_rows_tensor(const char* name, const void* p, int64_t ld, int64_t width, int e16)
{
    NA_CHECK(p, SOL_ERR_INVALID_ARGUMENT, "%s is NULL", name);
    NA_CHECK(aligned16(p), SOL_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
    NA_CHECK(ld >= width, SOL_ERR_INVALID_ARGUMENT, "ld of %s (%lld) is below the row width %lld", name,
             (long long)ld, (long long)width);
    NA_CHECK(ld % e16 == 0, SOL_ERR_MISALIGNED, "ld of %s (%lld) is not a multiple of %d elements",
             name, (long long)ld, e16);
    return SOL_OK;
}

// Element ranges of two [rows, width] tensors with row strides lda / ldb intersect?
bool overlaps(const void* a, int64_t lda, const void* b, int64_t ldb, int64_t rows, int64_t width,
              size_t esz)
{
    const char* a0 = (const char*)a;
    const char* b0 = (const char*)b;
    const char* a1 = a0 + (size_t)((rows - 1) * lda + width) * esz;
    const char* b1 = b0 + (size_t)((rows - 1) * ldb + width) * esz;
    return a0 < b1 && b0 < a1;
}

// Device address of the table for the current device (looked up once per device).
sol_status table_address(float2** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    NA_CHECK(e == cudaSuccess, SOL_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    NA_CHECK(dev >= 0 && dev < 64, SOL_ERR_UNSUPPORTED, "device index %d is out of range", dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_table_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_rope_noalloc_table);
        NA_CHECK(e == cudaSuccess && p, SOL_ERR_CUDA, "cudaGetSymbolAddress of the RoPE table: %s",
                 cudaGetErrorString(e));
        g_table_ptr[dev] = static_cast<float2*>(p);
    }
    *out = g_table_ptr[dev];
    return SOL_OK;
}

}  // namespace

extern "C" sol_status sol_qk_rmsnorm_rope3d_noalloc(
    void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
    int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
    int32_t grid_T, int32_t grid_H, int32_t grid_W, int64_t tokens_per_sample, int32_t dim_t,
    int32_t dim_h, int32_t dim_w, double theta, int32_t max_t, int32_t max_h, int32_t max_w,
    int64_t n_tokens, int32_t n_heads, int32_t head_dim, float eps, sol_dtype dt,
    sol_stream_t stream)
{
    NA_CHECK(dt == SOL_DTYPE_F32 || dt == SOL_DTYPE_BF16, SOL_ERR_UNSUPPORTED, "dtype %d is not built",
             (int)dt);
    const int e16 = dt == SOL_DTYPE_BF16 ? 8 : 4;
    const int32_t dims[3] = {dim_t, dim_h, dim_w};
    const int32_t maxp[3] = {max_t, max_h, max_w};
    for (int c = 0; c < 3; ++c) {
        NA_CHECK(dims[c] >= 0 && dims[c] % 2 == 0, SOL_ERR_INVALID_ARGUMENT,
                 "RoPE chunk width %d of axis %d must be even and >= 0", (int)dims[c], c);
        NA_CHECK(maxp[c] >= 1, SOL_ERR_INVALID_ARGUMENT, "max position of axis %d must be >= 1", c);
    }
    NA_CHECK(dim_t + dim_h + dim_w == head_dim, SOL_ERR_INVALID_ARGUMENT,
             "RoPE chunk widths (%d, %d, %d) do not sum to head_dim %d", (int)dim_t, (int)dim_h,
             (int)dim_w, (int)head_dim);
    NA_CHECK(std::isfinite(theta) && theta > 1.0, SOL_ERR_INVALID_ARGUMENT, "theta must be finite and > 1");
    const int64_t entries = (int64_t)max_t * (dim_t / 2) + (int64_t)max_h * (dim_h / 2) +
                            (int64_t)max_w * (dim_w / 2);
    NA_CHECK(entries <= kNoAllocRopeEntries, SOL_ERR_UNSUPPORTED,
             "the RoPE table needs %lld (cos, sin) entries; this entry point holds at most %lld "
             "(SOL_NOALLOC_MAX_ROPE_ENTRIES); use sol_qk_rmsnorm_rope3d with sol_rope3d_create",
             (long long)entries, (long long)kNoAllocRopeEntries);
    NA_CHECK(n_tokens >= 0, SOL_ERR_INVALID_ARGUMENT, "n_tokens is negative");
    NA_CHECK(n_heads >= 1 && n_heads <= 4096, SOL_ERR_INVALID_ARGUMENT, "n_heads (%d) must be in [1, 4096]",
             (int)n_heads);
    const int lph = head_dim / e16;
    NA_CHECK(head_dim % e16 == 0 && (lph == 8 || lph == 16 || lph == 32), SOL_ERR_UNSUPPORTED,
             "head_dim %d is not built for this dtype (bf16: 64/128/256, f32: 32/64/128)", (int)head_dim);
    NA_CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    NA_CHECK(!wq || aligned16(wq), SOL_ERR_MISALIGNED, "wq is not 16-byte aligned");
    NA_CHECK(!wk || aligned16(wk), SOL_ERR_MISALIGNED, "wk is not 16-byte aligned");
    NA_CHECK(tokens_per_sample >= 0, SOL_ERR_INVALID_ARGUMENT, "tokens_per_sample is negative");
    if (!pos) {
        NA_CHECK(grid_T >= 1 && grid_H >= 1 && grid_W >= 1, SOL_ERR_INVALID_ARGUMENT,
                 "implicit positions need grid_T, grid_H, grid_W >= 1");
        NA_CHECK(grid_T <= max_t && grid_H <= max_h && grid_W <= max_w, SOL_ERR_INVALID_ARGUMENT,
                 "grid %dx%dx%d exceeds the table extents (%d, %d, %d)", (int)grid_T, (int)grid_H,
                 (int)grid_W, (int)max_t, (int)max_h, (int)max_w);
        const int64_t span = tokens_per_sample > 0 ? tokens_per_sample : n_tokens;
        NA_CHECK(span <= (int64_t)grid_T * grid_H * grid_W, SOL_ERR_INVALID_ARGUMENT,
                 "%lld tokens per sample do not fit the grid", (long long)span);
    }
    if (n_tokens == 0) return SOL_OK;
    const int64_t hd = (int64_t)n_heads * head_dim;
    sol_status st;
    if ((st = check_rows_tensor("q", q, ld_q, hd, e16)) != SOL_OK) return st;
    if ((st = check_rows_tensor("k", k, ld_k, hd, e16)) != SOL_OK) return st;
    if ((st = check_rows_tensor("q_out", q_out, ld_qo, hd, e16)) != SOL_OK) return st;
    if ((st = check_rows_tensor("k_out", k_out, ld_ko, hd, e16)) != SOL_OK) return st;
    const size_t es = dt == SOL_DTYPE_BF16 ? 2 : 4;
    NA_CHECK(q_out == q ? ld_qo == ld_q : !overlaps(q_out, ld_qo, q, ld_q, n_tokens, hd, es),
             SOL_ERR_INVALID_ARGUMENT, "q_out overlaps q without being the same tensor");
    NA_CHECK(k_out == k ? ld_ko == ld_k : !overlaps(k_out, ld_ko, k, ld_k, n_tokens, hd, es),
             SOL_ERR_INVALID_ARGUMENT, "k_out overlaps k without being the same tensor");

    float2* table = nullptr;
    if ((st = table_address(&table)) != SOL_OK) return st;

    const cudaStream_t s = (cudaStream_t)stream;
    const int threads = 256;
    int64_t blocks = (entries + threads - 1) / threads;
    if (blocks > 1024) blocks = 1024;
    k_build_rope_table<<<(unsigned)blocks, threads, 0, s>>>(table, dim_t / 2, dim_h / 2, dim_w / 2,
                                                             max_t, max_h, max_w, theta);
    cudaError_t e = cudaGetLastError();
    NA_CHECK(e == cudaSuccess, SOL_ERR_CUDA, "RoPE table build launch: %s", cudaGetErrorString(e));

    sol::RopeDev view;
    view.tab[0] = table;
    view.tab[1] = table + (int64_t)max_t * (dim_t / 2);
    view.tab[2] = view.tab[1] + (int64_t)max_h * (dim_h / 2);
    for (int c = 0; c < 3; ++c) {
        view.max[c] = maxp[c];
        view.half[c] = dims[c] / 2;
    }
    e = sol::launch_qk_rmsnorm_rope3d(dt, q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k, wq, wk, pos,
                                      grid_T, grid_H, grid_W, tokens_per_sample, view, n_tokens,
                                      n_heads, head_dim, eps, s);
    NA_CHECK(e == cudaSuccess, SOL_ERR_CUDA, "sol_qk_rmsnorm_rope3d_noalloc launch: %s",
             cudaGetErrorString(e));
    return SOL_OK;
}
