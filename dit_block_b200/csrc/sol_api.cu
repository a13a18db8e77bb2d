// sol_api.cu -- the C ABI of libsol (declared in include/sol.h): argument validation,
// the RoPE table handle, launch bookkeeping, and dispatch to the kernel launchers.
// Every check runs on the host before anything is launched, so a rejected call has no
// side effect on the device.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <string>
#include <vector>

#include "common.cuh"
#include "launch.h"
#include "sol.h"

struct sol_rope3d {
    float2* dev;           // one allocation holding the three axis tables
    int32_t dims[3];       // chunk widths (t, h, w)
    int32_t max[3];        // positions per axis
    double theta;
    int device;
    sol::RopeDev view;
};

namespace {

thread_local std::string g_last_error;

sol_status fail(sol_status st, const char* fmt, ...)
{
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

sol_status cuda_status(cudaError_t e, const char* what)
{
    if (e == cudaSuccess) return SOL_OK;
    return fail(SOL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elems16(sol_dtype dt) { return dt == SOL_DTYPE_BF16 ? 8 : 4; }

#define CHECK(cond, st, ...)                      \
    do {                                          \
        if (!(cond)) return fail(st, __VA_ARGS__); \
    } while (0)

sol_status check_dtype(sol_dtype dt)
{
    CHECK(dt == SOL_DTYPE_F32 || dt == SOL_DTYPE_BF16, SOL_ERR_UNSUPPORTED,
          "dtype %d is not SOL_DTYPE_F32 or SOL_DTYPE_BF16", (int)dt);
    return SOL_OK;
}

// A required [rows, ld] tensor whose rows hold `width` used elements.
sol_status check_tensor(const char* name, const void* p, int64_t ld, int64_t width, sol_dtype dt,
                        bool required)
{
    if (!p) {
        CHECK(!required, SOL_ERR_INVALID_ARGUMENT, "%s is NULL", name);
        return SOL_OK;
    }
    CHECK(aligned16(p), SOL_ERR_MISALIGNED, "%s is not 16-byte aligned", name);
    CHECK(ld >= width, SOL_ERR_INVALID_ARGUMENT, "ld of %s (%lld) is below the row width %lld",
          name, (long long)ld, (long long)width);
    CHECK(ld % elems16(dt) == 0, SOL_ERR_MISALIGNED,
          "ld of %s (%lld) is not a multiple of %d elements (16 bytes)", name, (long long)ld,
          elems16(dt));
    return SOL_OK;
}

sol_status check_modsel(const sol_modsel& sel)
{
    CHECK(sel.n_streams >= 1 && sel.n_streams <= 256, SOL_ERR_INVALID_ARGUMENT,
          "sel.n_streams (%d) must be in [1, 256]", (int)sel.n_streams);
    CHECK(sel.tokens_per_sample >= 0, SOL_ERR_INVALID_ARGUMENT,
          "sel.tokens_per_sample (%lld) is negative", (long long)sel.tokens_per_sample);
    return SOL_OK;
}

sol::ModSel to_dev(const sol_modsel& sel, int64_t n_tokens)
{
    sol::ModSel m{sel.stream_id, sel.n_streams, sel.tokens_per_sample, 0u, 0u, 0};
    sol::modsel_prepare(m, n_tokens);
    return m;
}

// Do the element ranges of two [rows, width] tensors (row strides lda / ldb) overlap?
// A tensor spans from its first element to the end of its last row:
// ((rows - 1) * ld + width) elements.  Used to reject forbidden aliasing.
bool overlap(const void* a, int64_t lda, const void* b, int64_t ldb, int64_t rows, int64_t width,
             size_t esz)
{
    if (!a || !b || rows == 0) return false;
    const char* a0 = (const char*)a;
    const char* b0 = (const char*)b;
    const char* a1 = a0 + (size_t)((rows - 1) * lda + width) * esz;
    const char* b1 = b0 + (size_t)((rows - 1) * ldb + width) * esz;
    return a0 < b1 && b0 < a1;
}

size_t esize(sol_dtype dt) { return dt == SOL_DTYPE_BF16 ? 2 : 4; }

#define TRY(expr)                          \
    do {                                   \
        const sol_status st_ = (expr);     \
        if (st_ != SOL_OK) return st_;     \
    } while (0)

sol_status check_rows(int64_t n_tokens, int64_t d, sol_dtype dt, const char* dname)
{
    CHECK(n_tokens >= 0, SOL_ERR_INVALID_ARGUMENT, "n_tokens (%lld) is negative", (long long)n_tokens);
    CHECK(d >= elems16(dt), SOL_ERR_INVALID_ARGUMENT, "%s (%lld) is below %d", dname, (long long)d,
          elems16(dt));
    CHECK(d % elems16(dt) == 0, SOL_ERR_UNSUPPORTED, "%s (%lld) is not a multiple of %d", dname,
          (long long)d, elems16(dt));
    CHECK(d / elems16(dt) < (int64_t)1 << 30, SOL_ERR_UNSUPPORTED, "%s (%lld) is too wide", dname,
          (long long)d);
    return SOL_OK;
}

}  // namespace

namespace sol {

namespace {
struct OccEntry {
    const void* fn;
    int block;
    size_t smem;
    int device;
    int ctas;
};
std::mutex g_occ_mu;
std::vector<OccEntry> g_occ;
int g_sms[64];
}  // namespace

int ctas_per_sm(const void* kernel, int block, size_t smem)
{
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_occ_mu);
    for (const OccEntry& e : g_occ)
        if (e.fn == kernel && e.block == block && e.smem == smem && e.device == dev) return e.ctas;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, smem) != cudaSuccess || n < 1)
        n = 1;
    g_occ.push_back(OccEntry{kernel, block, smem, dev, n});
    return n;
}

void record_error(const char* msg) { g_last_error = msg; }

int sm_count()
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    std::lock_guard<std::mutex> lk(g_occ_mu);
    if (g_sms[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 1;
        g_sms[dev] = n;
    }
    return g_sms[dev];
}

}  // namespace sol

extern "C" {

const char* sol_status_string(sol_status status)
{
    switch (status) {
    case SOL_OK: return "ok";
    case SOL_ERR_INVALID_ARGUMENT: return "invalid argument";
    case SOL_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case SOL_ERR_UNSUPPORTED: return "unsupported configuration";
    case SOL_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char* sol_last_error(void) { return g_last_error.c_str(); }

int32_t sol_abi_version(void) { return 2; }

sol_status sol_device_errors(uint32_t* flags, int32_t clear)
{
    CHECK(flags, SOL_ERR_INVALID_ARGUMENT, "flags is NULL");
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e, "sol_device_errors");
    const uint32_t rows = sol::rows_device_error(clear != 0);
    const uint32_t staged = sol::rows_stage_device_error(clear != 0);
    const uint32_t qk = sol::qk_device_error(clear != 0);
    const uint32_t self = sol::selftest_device_error(clear != 0);
    CHECK(rows != 0xffffffffu && staged != 0xffffffffu && qk != 0xffffffffu && self != 0xffffffffu, SOL_ERR_CUDA,
          "reading the device error flags failed");
    *flags = rows | staged | qk | self | ((sol::gemm_device_error(clear != 0) & 0xffu) << 8);
    return SOL_OK;
}

sol_status sol_adaln_modulate(void* h, int64_t ld_h, const void* x, int64_t ld_x,
                              const void* shift, const void* scale, int64_t ld_mod,
                              sol_modsel sel, int64_t n_tokens, int64_t d, float eps,
                              sol_dtype dt, sol_stream_t stream)
{
    TRY(check_dtype(dt));
    TRY(check_rows(n_tokens, d, dt, "d"));
    CHECK(sol::adaln_row_fits(d / elems16(dt)), SOL_ERR_UNSUPPORTED,
          "d (%lld) is wider than one CTA row holds (max 4096 16-byte vectors)", (long long)d);
    CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    TRY(check_modsel(sel));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    TRY(check_tensor("h", h, ld_h, d, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    TRY(check_tensor("shift", shift, ld_mod, d, dt, false));
    TRY(check_tensor("scale", scale, ld_mod, d, dt, false));
    CHECK(h == x ? ld_h == ld_x : !overlap(h, ld_h, x, ld_x, n_tokens, d, esize(dt)),
          SOL_ERR_INVALID_ARGUMENT, "h overlaps x without being the same tensor");
    const sol::ModSel ms = to_dev(sel, n_tokens);
    return cuda_status(sol::launch_adaln_rows(dt, nullptr, 0, h, ld_h, x, ld_x, nullptr, 0, nullptr,
                                              shift, scale, ld_mod, ms, n_tokens, d, eps,
                                              (cudaStream_t)stream),
                       "sol_adaln_modulate launch");
}

sol_status sol_gated_residual(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                              const void* y, int64_t ld_y, const void* gate, int64_t ld_mod,
                              sol_modsel sel, int64_t n_tokens, int64_t d, sol_dtype dt,
                              sol_stream_t stream)
{
    TRY(check_dtype(dt));
    TRY(check_rows(n_tokens, d, dt, "d"));
    TRY(check_modsel(sel));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    TRY(check_tensor("out", out, ld_out, d, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    TRY(check_tensor("y", y, ld_y, d, dt, true));
    TRY(check_tensor("gate", gate, ld_mod, d, dt, false));
    CHECK(out == x ? ld_out == ld_x : !overlap(out, ld_out, x, ld_x, n_tokens, d, esize(dt)),
          SOL_ERR_INVALID_ARGUMENT, "out overlaps x without being the same tensor");
    CHECK(!overlap(out, ld_out, y, ld_y, n_tokens, d, esize(dt)), SOL_ERR_INVALID_ARGUMENT,
          "out overlaps y");
    const sol::ModSel ms = to_dev(sel, n_tokens);
    return cuda_status(sol::launch_gated_residual(dt, out, ld_out, x, ld_x, y, ld_y, gate, ld_mod,
                                                  ms, n_tokens, d, (cudaStream_t)stream),
                       "sol_gated_residual launch");
}

sol_status sol_gated_residual_cache_diff(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                         const void* y, int64_t ld_y, const void* gate,
                                         int64_t ld_mod, sol_modsel sel, void* cache,
                                         int64_t ld_cache, int32_t refresh, double* sums,
                                         int64_t n_samples, int64_t n_tokens, int64_t d,
                                         sol_dtype dt, sol_stream_t stream)
{
    TRY(check_dtype(dt));
    TRY(check_rows(n_tokens, d, dt, "d"));
    TRY(check_modsel(sel));
    CHECK(sums, SOL_ERR_INVALID_ARGUMENT, "sums is NULL");
    CHECK((reinterpret_cast<uintptr_t>(sums) & 7u) == 0, SOL_ERR_MISALIGNED, "sums is not 8-byte aligned");
    CHECK(n_samples >= 1, SOL_ERR_INVALID_ARGUMENT, "n_samples (%lld) must be >= 1", (long long)n_samples);
    const int64_t needed = sel.tokens_per_sample > 0
                               ? (n_tokens + sel.tokens_per_sample - 1) / sel.tokens_per_sample
                               : 1;
    CHECK(needed <= n_samples, SOL_ERR_INVALID_ARGUMENT,
          "%lld tokens at %lld per sample need %lld sample sums, n_samples is %lld",
          (long long)n_tokens, (long long)sel.tokens_per_sample, (long long)needed, (long long)n_samples);
    if (n_tokens > 0) {  // empty tensors may be NULL
        TRY(check_tensor("out", out, ld_out, d, dt, true));
        TRY(check_tensor("x", x, ld_x, d, dt, true));
        TRY(check_tensor("y", y, ld_y, d, dt, true));
        TRY(check_tensor("gate", gate, ld_mod, d, dt, false));
        TRY(check_tensor("cache", cache, ld_cache, d, dt, true));
        const size_t es = esize(dt);
        CHECK(out == x ? ld_out == ld_x : !overlap(out, ld_out, x, ld_x, n_tokens, d, es),
              SOL_ERR_INVALID_ARGUMENT, "out overlaps x without being the same tensor");
        CHECK(!overlap(out, ld_out, y, ld_y, n_tokens, d, es), SOL_ERR_INVALID_ARGUMENT, "out overlaps y");
        CHECK(!overlap(cache, ld_cache, out, ld_out, n_tokens, d, es) &&
                  !overlap(cache, ld_cache, x, ld_x, n_tokens, d, es) &&
                  !overlap(cache, ld_cache, y, ld_y, n_tokens, d, es),
              SOL_ERR_INVALID_ARGUMENT, "cache overlaps out, x or y");
    }
    // all arguments valid: clear the sums on the stream, then accumulate into them
    cudaError_t e = cudaMemsetAsync(sums, 0, (size_t)n_samples * 2 * sizeof(double), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e, "sol_gated_residual_cache_diff clearing sums");
    if (n_tokens == 0) return SOL_OK;
    const sol::ModSel ms = to_dev(sel, n_tokens);
    return cuda_status(sol::launch_gated_residual_diff(dt, out, ld_out, x, ld_x, y, ld_y, gate, ld_mod,
                                                       cache, ld_cache, refresh != 0, sums, ms,
                                                       n_tokens, d, (cudaStream_t)stream),
                       "sol_gated_residual_cache_diff launch");
}

sol_status sol_swiglu(void* out, int64_t ld_out, const void* a, const void* b, int64_t ld_in,
                      int64_t n_tokens, int64_t inner, sol_dtype dt, sol_stream_t stream)
{
    TRY(check_dtype(dt));
    TRY(check_rows(n_tokens, inner, dt, "inner"));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    TRY(check_tensor("out", out, ld_out, inner, dt, true));
    TRY(check_tensor("a", a, ld_in, inner, dt, true));
    TRY(check_tensor("b", b, ld_in, inner, dt, true));
    // a and b may be two halves of one row: the row extent of each is ld_in wide
    CHECK(!overlap(out, ld_out, a, ld_in, n_tokens, inner, esize(dt)) &&
              !overlap(out, ld_out, b, ld_in, n_tokens, inner, esize(dt)),
          SOL_ERR_INVALID_ARGUMENT, "out overlaps a or b");
    return cuda_status(sol::launch_swiglu(dt, out, ld_out, a, b, ld_in, n_tokens, inner,
                                          (cudaStream_t)stream),
                       "sol_swiglu launch");
}

sol_status sol_rope3d_create(sol_rope3d** out, int32_t dim_t, int32_t dim_h, int32_t dim_w,
                             double theta, int32_t max_t, int32_t max_h, int32_t max_w)
{
    CHECK(out, SOL_ERR_INVALID_ARGUMENT, "out is NULL");
    *out = nullptr;
    const int32_t dims[3] = {dim_t, dim_h, dim_w};
    const int32_t maxp[3] = {max_t, max_h, max_w};
    for (int c = 0; c < 3; ++c) {
        CHECK(dims[c] >= 0 && dims[c] % 2 == 0 && dims[c] <= 1024, SOL_ERR_INVALID_ARGUMENT,
              "RoPE chunk width %d of axis %d must be even and in [0, 1024]", (int)dims[c], c);
        CHECK(maxp[c] >= 1 && maxp[c] <= (1 << 20), SOL_ERR_INVALID_ARGUMENT,
              "max position %d of axis %d must be in [1, 2^20]", (int)maxp[c], c);
    }
    CHECK(dim_t + dim_h + dim_w >= 2, SOL_ERR_INVALID_ARGUMENT, "RoPE chunk widths sum to 0");
    CHECK(std::isfinite(theta) && theta > 1.0, SOL_ERR_INVALID_ARGUMENT, "theta must be finite and > 1");

    size_t off[4] = {0, 0, 0, 0};
    for (int c = 0; c < 3; ++c) off[c + 1] = off[c] + (size_t)maxp[c] * (size_t)(dims[c] / 2);
    // tables on the host in fp64, rounded once to fp32: phi = p * theta^(-2j/D_c)
    std::vector<float2> host(off[3] > 0 ? off[3] : 1);
    for (int c = 0; c < 3; ++c) {
        const int half = dims[c] / 2;
        for (int32_t p = 0; p < maxp[c]; ++p) {
            for (int j = 0; j < half; ++j) {
                const double inv_freq = std::pow(theta, -2.0 * (double)j / (double)dims[c]);
                const double phi = (double)p * inv_freq;
                host[off[c] + (size_t)p * half + j] = make_float2((float)std::cos(phi), (float)std::sin(phi));
            }
        }
    }
    sol_rope3d* r = new (std::nothrow) sol_rope3d();
    CHECK(r, SOL_ERR_INVALID_ARGUMENT, "host allocation failed");
    cudaGetDevice(&r->device);
    cudaError_t e = cudaMalloc((void**)&r->dev, host.size() * sizeof(float2));
    if (e != cudaSuccess) {
        delete r;
        return cuda_status(e, "sol_rope3d_create cudaMalloc");
    }
    e = cudaMemcpy(r->dev, host.data(), host.size() * sizeof(float2), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(r->dev);
        delete r;
        return cuda_status(e, "sol_rope3d_create cudaMemcpy");
    }
    for (int c = 0; c < 3; ++c) {
        r->dims[c] = dims[c];
        r->max[c] = maxp[c];
        r->view.tab[c] = r->dev + off[c];
        r->view.max[c] = maxp[c];
        r->view.half[c] = dims[c] / 2;
    }
    r->theta = theta;
    *out = r;
    return SOL_OK;
}

sol_status sol_rope3d_destroy(sol_rope3d* rope)
{
    if (!rope) return SOL_OK;
    const cudaError_t e = cudaFree(rope->dev);
    delete rope;
    return cuda_status(e, "sol_rope3d_destroy cudaFree");
}

static sol_status check_qk_common(const sol_rope3d* rope, const int32_t* pos, int32_t grid_T,
                                  int32_t grid_H, int32_t grid_W, int64_t tps, int64_t n_tokens,
                                  int32_t n_heads, int32_t head_dim, float eps, sol_dtype dt,
                                  const void* wq, const void* wk)
{
    TRY(check_dtype(dt));
    CHECK(rope, SOL_ERR_INVALID_ARGUMENT, "rope is NULL");
    CHECK(n_tokens >= 0, SOL_ERR_INVALID_ARGUMENT, "n_tokens is negative");
    CHECK(n_heads >= 1 && n_heads <= 4096, SOL_ERR_INVALID_ARGUMENT, "n_heads (%d) must be in [1, 4096]",
          (int)n_heads);
    const int lph = head_dim / elems16(dt);
    CHECK(head_dim % elems16(dt) == 0 && (lph == 8 || lph == 16 || lph == 32), SOL_ERR_UNSUPPORTED,
          "head_dim %d is not built for this dtype (bf16: 64/128/256, f32: 32/64/128)", (int)head_dim);
    CHECK(rope->dims[0] + rope->dims[1] + rope->dims[2] == head_dim, SOL_ERR_INVALID_ARGUMENT,
          "RoPE chunk widths (%d, %d, %d) do not sum to head_dim %d", (int)rope->dims[0],
          (int)rope->dims[1], (int)rope->dims[2], (int)head_dim);
    CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    CHECK(!wq || aligned16(wq), SOL_ERR_MISALIGNED, "wq is not 16-byte aligned");
    CHECK(!wk || aligned16(wk), SOL_ERR_MISALIGNED, "wk is not 16-byte aligned");
    CHECK(tps >= 0, SOL_ERR_INVALID_ARGUMENT, "tokens_per_sample is negative");
    if (!pos) {
        CHECK(grid_T >= 1 && grid_H >= 1 && grid_W >= 1, SOL_ERR_INVALID_ARGUMENT,
              "implicit positions need grid_T, grid_H, grid_W >= 1");
        CHECK(grid_T <= rope->max[0] && grid_H <= rope->max[1] && grid_W <= rope->max[2],
              SOL_ERR_INVALID_ARGUMENT, "grid %dx%dx%d exceeds the RoPE tables (%d, %d, %d)",
              (int)grid_T, (int)grid_H, (int)grid_W, (int)rope->max[0], (int)rope->max[1],
              (int)rope->max[2]);
        const int64_t cells = (int64_t)grid_T * grid_H * grid_W;
        const int64_t span = tps > 0 ? tps : n_tokens;
        CHECK(span <= cells, SOL_ERR_INVALID_ARGUMENT,
              "%lld tokens per sample do not fit the %lld-cell grid", (long long)span, (long long)cells);
    }
    int dev = 0;
    cudaGetDevice(&dev);
    CHECK(dev == rope->device, SOL_ERR_INVALID_ARGUMENT,
          "rope tables live on device %d, current device is %d", rope->device, dev);
    return SOL_OK;
}

sol_status sol_qk_rmsnorm_rope3d(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko,
                                 const void* q, const void* k, int64_t ld_q, int64_t ld_k,
                                 const void* wq, const void* wk, const int32_t* pos,
                                 int32_t grid_T, int32_t grid_H, int32_t grid_W,
                                 int64_t tokens_per_sample, const sol_rope3d* rope,
                                 int64_t n_tokens, int32_t n_heads, int32_t head_dim, float eps,
                                 sol_dtype dt, sol_stream_t stream)
{
    TRY(check_qk_common(rope, pos, grid_T, grid_H, grid_W, tokens_per_sample, n_tokens, n_heads,
                        head_dim, eps, dt, wq, wk));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    const int64_t hd = (int64_t)n_heads * head_dim;
    TRY(check_tensor("q", q, ld_q, hd, dt, true));
    TRY(check_tensor("k", k, ld_k, hd, dt, true));
    TRY(check_tensor("q_out", q_out, ld_qo, hd, dt, true));
    TRY(check_tensor("k_out", k_out, ld_ko, hd, dt, true));
    const size_t es = esize(dt);
    CHECK(q_out == q ? ld_qo == ld_q : !overlap(q_out, ld_qo, q, ld_q, n_tokens, hd, es),
          SOL_ERR_INVALID_ARGUMENT, "q_out overlaps q without being the same tensor");
    CHECK(k_out == k ? ld_ko == ld_k : !overlap(k_out, ld_ko, k, ld_k, n_tokens, hd, es),
          SOL_ERR_INVALID_ARGUMENT, "k_out overlaps k without being the same tensor");
    return cuda_status(sol::launch_qk_rmsnorm_rope3d(dt, q_out, k_out, ld_qo, ld_ko, q, k, ld_q, ld_k,
                                                     wq, wk, pos, grid_T, grid_H, grid_W,
                                                     tokens_per_sample, rope->view, n_tokens,
                                                     n_heads, head_dim, eps, (cudaStream_t)stream),
                       "sol_qk_rmsnorm_rope3d launch");
}

sol_status sol_qk_rmsnorm_rope3d_ex(const sol_qk_desc* d, sol_stream_t stream)
{
    CHECK(d, SOL_ERR_INVALID_ARGUMENT, "desc is NULL");
    TRY(check_qk_common(d->rope, d->pos, d->grid_T, d->grid_H, d->grid_W, d->tokens_per_sample, d->n_tokens,
                        d->n_heads, d->head_dim, d->eps, d->dt, d->wq, d->wk));
    CHECK(d->norm_span == SOL_NORM_PER_HEAD || d->norm_span == SOL_NORM_ACROSS_HEADS, SOL_ERR_INVALID_ARGUMENT,
          "norm_span %d is not a sol_norm_span", (int)d->norm_span);
    CHECK(d->rope_pairing == SOL_ROPE_INTERLEAVED || d->rope_pairing == SOL_ROPE_HALF, SOL_ERR_INVALID_ARGUMENT,
          "rope_pairing %d is not a sol_rope_pairing", (int)d->rope_pairing);
    const int e16 = elems16(d->dt);
    if (d->rope_pairing == SOL_ROPE_HALF)
        for (int c = 0; c < 3; ++c)
            CHECK(d->rope->dims[c] % (2 * e16) == 0, SOL_ERR_UNSUPPORTED,
                  "rotate-half pairing needs chunk widths that are multiples of %d (chunk %d is %d)", 2 * e16, c,
                  (int)d->rope->dims[c]);
    const int64_t ts = d->out_token_stride, hs = d->out_head_stride, ss = d->out_sample_stride;
    CHECK(ts > 0 && hs > 0 && ss >= 0, SOL_ERR_INVALID_ARGUMENT, "output strides must be positive");
    CHECK(ts % e16 == 0 && hs % e16 == 0 && ss % e16 == 0, SOL_ERR_MISALIGNED,
          "output strides must be multiples of %d elements", e16);
    if (d->n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    const int64_t hd = (int64_t)d->n_heads * d->head_dim;
    TRY(check_tensor("q", d->q, d->ld_q, hd, d->dt, true));
    TRY(check_tensor("k", d->k, d->ld_k, hd, d->dt, true));
    CHECK(d->q_out && d->k_out, SOL_ERR_INVALID_ARGUMENT, "q_out or k_out is NULL");
    CHECK(aligned16(d->q_out) && aligned16(d->k_out), SOL_ERR_MISALIGNED, "q_out or k_out is not 16-byte aligned");
    // extent of an output: the farthest element it addresses, plus one
    const int64_t tps = d->tokens_per_sample > 0 ? d->tokens_per_sample : d->n_tokens;
    const int64_t n_samples = (d->n_tokens + tps - 1) / tps;
    const int64_t last_local = d->n_tokens <= tps ? d->n_tokens - 1 : tps - 1;
    const int64_t extent = (n_samples - 1) * ss + last_local * ts + (int64_t)(d->n_heads - 1) * hs + d->head_dim;
    const size_t es = esize(d->dt);
    auto range_overlap = [&](const void* a, int64_t na, const void* b, int64_t nb) {
        const char* a0 = (const char*)a;
        const char* b0 = (const char*)b;
        return a0 < b0 + nb * (int64_t)es && b0 < a0 + na * (int64_t)es;
    };
    const int64_t in_q = (d->n_tokens - 1) * d->ld_q + hd, in_k = (d->n_tokens - 1) * d->ld_k + hd;
    const bool token_major_q = ts == d->ld_q && hs == d->head_dim && (ss == tps * d->ld_q || n_samples == 1);
    const bool token_major_k = ts == d->ld_k && hs == d->head_dim && (ss == tps * d->ld_k || n_samples == 1);
    CHECK(d->q_out == d->q ? token_major_q : !range_overlap(d->q_out, extent, d->q, in_q) && !range_overlap(d->q_out, extent, d->k, in_k),
          SOL_ERR_INVALID_ARGUMENT, "q_out overlaps the inputs other than as q itself with q's layout");
    CHECK(d->k_out == d->k ? token_major_k : !range_overlap(d->k_out, extent, d->k, in_k) && !range_overlap(d->k_out, extent, d->q, in_q),
          SOL_ERR_INVALID_ARGUMENT, "k_out overlaps the inputs other than as k itself with k's layout");
    CHECK(!range_overlap(d->q_out, extent, d->k_out, extent) || (d->q_out == d->q && d->k_out == d->k),
          SOL_ERR_INVALID_ARGUMENT, "q_out and k_out overlap");
    const sol::QkOutStrides os{ts, hs, ss};
    return cuda_status(sol::launch_qk_ex(d->dt, d->norm_span == SOL_NORM_ACROSS_HEADS,
                                         d->rope_pairing == SOL_ROPE_HALF, d->q_out, d->k_out, os, d->q, d->k,
                                         d->ld_q, d->ld_k, d->wq, d->wk, d->pos, d->grid_H, d->grid_W,
                                         d->tokens_per_sample, d->rope->view, d->n_tokens, d->n_heads,
                                         d->head_dim, d->eps, (cudaStream_t)stream),
                       "sol_qk_rmsnorm_rope3d_ex launch");
}

sol_status sol_dit_prologue(void* x_out, void* h, const void* x, const void* y,
                            const void* gate, const void* shift, const void* scale, int64_t ld,
                            int64_t ld_mod, sol_modsel sel, int64_t n_tokens, int64_t d,
                            float eps, sol_dtype dt, sol_stream_t stream)
{
    TRY(check_dtype(dt));
    TRY(check_rows(n_tokens, d, dt, "d"));
    CHECK(sol::adaln_row_fits(d / elems16(dt)), SOL_ERR_UNSUPPORTED,
          "d (%lld) is wider than one CTA row holds (max 4096 16-byte vectors)", (long long)d);
    CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    TRY(check_modsel(sel));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    TRY(check_tensor("h", h, ld, d, dt, true));
    TRY(check_tensor("x", x, ld, d, dt, true));
    TRY(check_tensor("y", y, ld, d, dt, false));
    TRY(check_tensor("x_out", x_out, ld, d, dt, y != nullptr));
    TRY(check_tensor("gate", gate, ld_mod, d, dt, false));
    TRY(check_tensor("shift", shift, ld_mod, d, dt, false));
    TRY(check_tensor("scale", scale, ld_mod, d, dt, false));
    const size_t es = esize(dt);
    CHECK(!overlap(h, ld, x, ld, n_tokens, d, es) && !overlap(h, ld, y, ld, n_tokens, d, es) &&
              !overlap(h, ld, x_out, ld, n_tokens, d, es),
          SOL_ERR_INVALID_ARGUMENT, "h overlaps x, y or x_out");
    CHECK(!y || x_out == x || !overlap(x_out, ld, x, ld, n_tokens, d, es), SOL_ERR_INVALID_ARGUMENT,
          "x_out overlaps x without being the same tensor");
    CHECK(!y || !overlap(x_out, ld, y, ld, n_tokens, d, es), SOL_ERR_INVALID_ARGUMENT, "x_out overlaps y");
    const sol::ModSel ms = to_dev(sel, n_tokens);
    return cuda_status(sol::launch_adaln_rows(dt, y ? x_out : nullptr, ld, h, ld, x, ld, y, ld, gate,
                                              shift, scale, ld_mod, ms, n_tokens, d, eps,
                                              (cudaStream_t)stream),
                       "sol_dit_prologue launch");
}

int64_t sol_subblock_count(int64_t n_tokens, int64_t tokens_per_sample, int32_t block_tokens)
{
    if (n_tokens <= 0 || block_tokens <= 0 || tokens_per_sample < 0) return 0;
    const int64_t tps = tokens_per_sample > 0 ? tokens_per_sample : n_tokens;
    const int64_t samples = (n_tokens + tps - 1) / tps;
    return samples * ((tps + block_tokens - 1) / block_tokens);
}

sol_status sol_dit_epilogue_pool(void* qkv, int64_t ld_qkv, const void* wq, const void* wk,
                                 const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                                 int64_t tokens_per_sample, const sol_rope3d* rope, int64_t n_tokens,
                                 int32_t n_heads, int32_t head_dim, float eps, void* pooled_q,
                                 void* pooled_k, int64_t ld_pool, int32_t block_tokens, sol_dtype dt,
                                 sol_stream_t stream)
{
    TRY(check_qk_common(rope, pos, grid_T, grid_H, grid_W, tokens_per_sample, n_tokens, n_heads,
                        head_dim, eps, dt, wq, wk));
    CHECK(block_tokens >= 1 && block_tokens <= (1 << 20), SOL_ERR_INVALID_ARGUMENT,
          "block_tokens (%d) must be in [1, 2^20]", (int)block_tokens);
    CHECK(sol::qk_pool_smem_bytes(dt, n_heads, head_dim) <= sol::qk_pool_smem_limit(), SOL_ERR_UNSUPPORTED,
          "%d heads of %d need a larger block accumulator than the pooled epilogue holds", (int)n_heads,
          (int)head_dim);
    if (n_tokens == 0) return SOL_OK;  // nothing to do; empty tensors may be NULL
    const int64_t hd = (int64_t)n_heads * head_dim;
    TRY(check_tensor("qkv", qkv, ld_qkv, 2 * hd, dt, true));
    const int64_t n_blocks = sol_subblock_count(n_tokens, tokens_per_sample, block_tokens);
    TRY(check_tensor("pooled_q", pooled_q, ld_pool, hd, dt, true));
    TRY(check_tensor("pooled_k", pooled_k, ld_pool, hd, dt, true));
    const size_t es = esize(dt);
    CHECK(!overlap(pooled_q, ld_pool, pooled_k, ld_pool, n_blocks, hd, es) &&
              !overlap(pooled_q, ld_pool, qkv, ld_qkv, n_blocks < n_tokens ? n_blocks : n_tokens, hd, es) &&
              !overlap(pooled_k, ld_pool, qkv, ld_qkv, n_blocks < n_tokens ? n_blocks : n_tokens, hd, es),
          SOL_ERR_INVALID_ARGUMENT, "pooled outputs overlap each other or qkv");
    const int64_t tps = tokens_per_sample > 0 ? tokens_per_sample : n_tokens;
    const int64_t bps = (tps + block_tokens - 1) / block_tokens;
    void* k = (char*)qkv + (size_t)hd * es;
    return cuda_status(sol::launch_qk_rope_pool(dt, qkv, k, ld_qkv, ld_qkv, pooled_q, pooled_k, ld_pool,
                                                ld_pool, wq, wk, pos, grid_H, grid_W, tps, block_tokens,
                                                bps, n_blocks, rope->view, n_tokens, n_heads, head_dim,
                                                eps, (cudaStream_t)stream),
                       "sol_dit_epilogue_pool launch");
}

sol_status sol_dit_epilogue(void* qkv, int64_t ld_qkv, const void* wq, const void* wk,
                            const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                            int64_t tokens_per_sample, const sol_rope3d* rope, int64_t n_tokens,
                            int32_t n_heads, int32_t head_dim, float eps, sol_dtype dt,
                            sol_stream_t stream)
{
    TRY(check_qk_common(rope, pos, grid_T, grid_H, grid_W, tokens_per_sample, n_tokens, n_heads,
                        head_dim, eps, dt, wq, wk));
    if (n_tokens == 0) return SOL_OK;  // nothing to do; an empty tensor may be NULL
    const int64_t hd = (int64_t)n_heads * head_dim;
    TRY(check_tensor("qkv", qkv, ld_qkv, 2 * hd, dt, true));
    void* k = (char*)qkv + (size_t)hd * esize(dt);
    return cuda_status(sol::launch_qk_rmsnorm_rope3d(dt, qkv, k, ld_qkv, ld_qkv, qkv, k, ld_qkv,
                                                     ld_qkv, wq, wk, pos, grid_T, grid_H, grid_W,
                                                     tokens_per_sample, rope->view, n_tokens,
                                                     n_heads, head_dim, eps, (cudaStream_t)stream),
                       "sol_dit_epilogue launch");
}

}  // extern "C"

// Shared checks of the linear-layer calls: bf16 only, k a multiple of 64, n_out a
// multiple of 256, n_tokens below 2^31 (tensor-copy coordinates are 32-bit).
static sol_status check_linear_shape(int64_t n_tokens, int64_t n_out, int64_t k, sol_dtype dt,
                                     int64_t n_multiple)
{
    CHECK(dt == SOL_DTYPE_BF16, SOL_ERR_UNSUPPORTED, "the linear-layer calls take bf16 only");
    CHECK(n_tokens >= 0, SOL_ERR_INVALID_ARGUMENT, "n_tokens (%lld) is negative", (long long)n_tokens);
    CHECK(n_tokens < ((int64_t)1 << 31), SOL_ERR_UNSUPPORTED, "n_tokens (%lld) must be below 2^31",
          (long long)n_tokens);
    CHECK(k >= 64 && n_out >= 1, SOL_ERR_INVALID_ARGUMENT, "k (%lld) and the output width (%lld) must be positive, k >= 64",
          (long long)k, (long long)n_out);
    CHECK(k % 64 == 0 && k < ((int64_t)1 << 30), SOL_ERR_UNSUPPORTED, "k (%lld) must be a multiple of 64",
          (long long)k);
    CHECK(n_out % n_multiple == 0 && n_out < ((int64_t)1 << 30), SOL_ERR_UNSUPPORTED,
          "output width %lld must be a multiple of %lld", (long long)n_out, (long long)n_multiple);
    return SOL_OK;
}

// Byte-range overlap of two row-strided tensors of different shapes.
// Element sizes: esz_a for a, esz_b for b.
static bool spans_overlap(const void* a, int64_t rows_a, int64_t ld_a, int64_t w_a, size_t esz_a, const void* b,
                          int64_t rows_b, int64_t ld_b, int64_t w_b, size_t esz_b)
{
    if (!a || !b || rows_a == 0 || rows_b == 0) return false;
    const char* a0 = (const char*)a;
    const char* b0 = (const char*)b;
    const char* a1 = a0 + (size_t)((rows_a - 1) * ld_a + w_a) * esz_a;
    const char* b1 = b0 + (size_t)((rows_b - 1) * ld_b + w_b) * esz_b;
    return a0 < b1 && b0 < a1;
}

// Modulation rows a call may use: ceil(n_tokens / tokens_per_sample) * n_streams, or
// n_streams for one sample.
static int64_t mod_rows(int64_t n_tokens, const sol_modsel& sel)
{
    const int64_t samples = sel.tokens_per_sample > 0 ? (n_tokens + sel.tokens_per_sample - 1) / sel.tokens_per_sample : 1;
    return std::max<int64_t>(samples, 1) * sel.n_streams;
}

// Workspace of the sol_adaln_* calls: row statistics, per-128-row modulation-row sets,
// folded-weight column sums and shift projections, then one region that holds either the
// folded weights (fold strategy) or the staged AdaLN output h (stage strategy), whichever
// is larger; every region 256-byte aligned.
struct AdalnWorkspace {
    size_t stats, rmask, c, b, v, total;
};

static AdalnWorkspace adaln_layout(int64_t n_tokens, int64_t n_out, int64_t d, int64_t R)
{
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    AdalnWorkspace w{};
    w.stats = 0;
    w.rmask = up(w.stats + (size_t)n_tokens * 8);
    w.c = up(w.rmask + (size_t)((n_tokens + 127) / 128) * 4);
    w.b = up(w.c + (size_t)(R * n_out) * 4);
    w.v = up(w.b + (size_t)(R * n_out) * 4);
    const size_t folded = (size_t)(R * n_out) * (size_t)d * 2, staged = (size_t)n_tokens * (size_t)d * 2;
    w.total = up(w.v + (folded > staged ? folded : staged));
    return w;
}

static sol_status check_workspace(const void* ws, size_t bytes, int64_t n_tokens, int64_t n_out, int64_t d,
                                  const sol_modsel& sel, AdalnWorkspace* lay, int64_t* R)
{
    *R = mod_rows(n_tokens, sel);
    CHECK(*R <= 32, SOL_ERR_UNSUPPORTED, "%lld modulation rows (more than 32)", (long long)*R);
    *lay = adaln_layout(n_tokens, n_out, d, *R);
    CHECK(ws, SOL_ERR_INVALID_ARGUMENT, "workspace is NULL");
    CHECK((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, SOL_ERR_MISALIGNED, "workspace is not 256-byte aligned");
    CHECK(bytes >= lay->total, SOL_ERR_INVALID_ARGUMENT, "workspace of %zu bytes is below the %zu needed", bytes,
          lay->total);
    return SOL_OK;
}

static sol_status check_strategy(int32_t strategy)
{
    CHECK(strategy == SOL_ADALN_STAGE || strategy == SOL_ADALN_FOLD || strategy == SOL_ADALN_TRANSFORM,
          SOL_ERR_INVALID_ARGUMENT, "strategy %d is not a sol_adaln_strategy", (int)strategy);
    return SOL_OK;
}

static void set_workspace(sol::LinearLaunch& L, void* ws, const AdalnWorkspace& lay, int64_t R)
{
    char* base = static_cast<char*>(ws);
    L.stats = base + lay.stats;
    L.rmask = reinterpret_cast<uint32_t*>(base + lay.rmask);
    L.fold_c = reinterpret_cast<float*>(base + lay.c);
    L.fold_b = reinterpret_cast<float*>(base + lay.b);
    L.fold_v = base + lay.v;
    L.n_mod_rows = (int32_t)R;
}

static sol::LinearLaunch linear_base(void* out, int64_t ld_out, const void* a, int64_t ld_a, const void* w,
                                     int64_t ld_w, int64_t n_tokens, int64_t n_w_rows, int64_t k)
{
    sol::LinearLaunch L{};
    L.M = n_tokens;
    L.K = (int32_t)k;
    L.N = (int32_t)n_w_rows;
    L.a = a;
    L.ld_a = ld_a;
    L.w = w;
    L.ld_w = ld_w;
    L.out = out;
    L.ld_out = ld_out;
    L.eps = 0.f;
    return L;
}

extern "C" {

sol_status sol_linear(void* out, int64_t ld_out, const void* a, int64_t ld_a, const void* w,
                      int64_t ld_w, int64_t n_tokens, int64_t n_out, int64_t k, sol_dtype dt,
                      sol_stream_t stream)
{
    TRY(check_linear_shape(n_tokens, n_out, k, dt, 256));
    TRY(check_tensor("w", w, ld_w, k, dt, true));
    if (n_tokens == 0) return SOL_OK;
    TRY(check_tensor("out", out, ld_out, n_out, dt, true));
    TRY(check_tensor("a", a, ld_a, k, dt, true));
    CHECK(!spans_overlap(out, n_tokens, ld_out, n_out, 2, a, n_tokens, ld_a, k, 2) &&
              !spans_overlap(out, n_tokens, ld_out, n_out, 2, w, n_out, ld_w, k, 2),
          SOL_ERR_INVALID_ARGUMENT, "out overlaps an input");
    const sol::LinearLaunch L = linear_base(out, ld_out, a, ld_a, w, ld_w, n_tokens, n_out, k);
    return cuda_status(sol::launch_linear(sol::LINEAR_STORE, false, L, (cudaStream_t)stream), "sol_linear launch");
}

sol_status sol_linear_gated_residual(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                     const void* a, int64_t ld_a, const void* w, int64_t ld_w,
                                     const void* gate, int64_t ld_mod, sol_modsel sel,
                                     int64_t n_tokens, int64_t d, int64_t k, sol_dtype dt,
                                     sol_stream_t stream)
{
    TRY(check_linear_shape(n_tokens, d, k, dt, 256));
    TRY(check_modsel(sel));
    TRY(check_tensor("w", w, ld_w, k, dt, true));
    TRY(check_tensor("gate", gate, ld_mod, d, dt, false));
    if (n_tokens == 0) return SOL_OK;
    TRY(check_tensor("out", out, ld_out, d, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    TRY(check_tensor("a", a, ld_a, k, dt, true));
    CHECK(out == x ? ld_out == ld_x : !overlap(out, ld_out, x, ld_x, n_tokens, d, 2), SOL_ERR_INVALID_ARGUMENT,
          "out overlaps x without being the same tensor");
    CHECK(!spans_overlap(out, n_tokens, ld_out, d, 2, a, n_tokens, ld_a, k, 2) &&
              !spans_overlap(out, n_tokens, ld_out, d, 2, w, d, ld_w, k, 2),
          SOL_ERR_INVALID_ARGUMENT, "out overlaps a or w");
    sol::LinearLaunch L = linear_base(out, ld_out, a, ld_a, w, ld_w, n_tokens, d, k);
    const sol::ModSel ms = to_dev(sel, n_tokens);
    L.x = x;
    L.ld_x = ld_x;
    L.gate = gate;
    L.ld_mod = ld_mod;
    L.sel = &ms;
    return cuda_status(sol::launch_linear(sol::LINEAR_GATED, false, L, (cudaStream_t)stream),
                       "sol_linear_gated_residual launch");
}

sol_status sol_linear_swiglu(void* out, int64_t ld_out, const void* a, int64_t ld_a, const void* w,
                             int64_t ld_w, int64_t n_tokens, int64_t inner, int64_t k, sol_dtype dt,
                             sol_stream_t stream)
{
    TRY(check_linear_shape(n_tokens, 2 * inner, k, dt, 256));
    TRY(check_tensor("w", w, ld_w, k, dt, true));
    if (n_tokens == 0) return SOL_OK;
    TRY(check_tensor("out", out, ld_out, inner, dt, true));
    TRY(check_tensor("a", a, ld_a, k, dt, true));
    CHECK(!spans_overlap(out, n_tokens, ld_out, inner, 2, a, n_tokens, ld_a, k, 2) &&
              !spans_overlap(out, n_tokens, ld_out, inner, 2, w, 2 * inner, ld_w, k, 2),
          SOL_ERR_INVALID_ARGUMENT, "out overlaps a or w");
    const sol::LinearLaunch L = linear_base(out, ld_out, a, ld_a, w, ld_w, n_tokens, 2 * inner, k);
    return cuda_status(sol::launch_linear(sol::LINEAR_SWIGLU, false, L, (cudaStream_t)stream),
                       "sol_linear_swiglu launch");
}

size_t sol_adaln_workspace_bytes(int64_t n_tokens, int64_t n_out, int64_t d, sol_modsel sel)
{
    if (n_tokens < 0 || n_out < 1 || d < 1 || sel.n_streams < 1 || sel.tokens_per_sample < 0) return 0;
    const int64_t R = mod_rows(n_tokens, sel);
    if (R > 32) return 0;
    return adaln_layout(n_tokens, n_out, d, R).total;
}

sol_status sol_adaln_linear(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                            const void* shift, const void* scale, int64_t ld_mod, sol_modsel sel,
                            const void* w, int64_t ld_w, void* workspace, size_t workspace_bytes,
                            int32_t strategy, int64_t n_tokens, int64_t n_out, int64_t d, float eps,
                            sol_dtype dt, sol_stream_t stream)
{
    TRY(check_strategy(strategy));
    TRY(check_linear_shape(n_tokens, n_out, d, dt, 256));
    TRY(check_modsel(sel));
    CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    TRY(check_tensor("w", w, ld_w, d, dt, true));
    TRY(check_tensor("shift", shift, ld_mod, d, dt, false));
    TRY(check_tensor("scale", scale, ld_mod, d, dt, false));
    if (n_tokens == 0) return SOL_OK;
    AdalnWorkspace lay;
    int64_t R = 0;
    TRY(check_workspace(workspace, workspace_bytes, n_tokens, n_out, d, sel, &lay, &R));
    TRY(check_tensor("out", out, ld_out, n_out, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    CHECK(!spans_overlap(out, n_tokens, ld_out, n_out, 2, x, n_tokens, ld_x, d, 2) &&
              !spans_overlap(out, n_tokens, ld_out, n_out, 2, w, n_out, ld_w, d, 2) &&
              !spans_overlap(out, n_tokens, ld_out, n_out, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(x, n_tokens, ld_x, d, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(w, n_out, ld_w, d, 2, workspace, 1, 0, (int64_t)lay.total, 1),
          SOL_ERR_INVALID_ARGUMENT, "out, x or w overlaps another argument");
    sol::LinearLaunch L = linear_base(out, ld_out, x, ld_x, w, ld_w, n_tokens, n_out, d);
    const sol::ModSel ms = to_dev(sel, n_tokens);
    set_workspace(L, workspace, lay, R);
    L.shift = shift;
    L.scale = scale;
    L.ld_mod = ld_mod;
    L.sel = &ms;
    L.eps = eps;
    L.adaln_strategy = strategy;
    return cuda_status(sol::launch_linear(sol::LINEAR_STORE, true, L, (cudaStream_t)stream),
                       "sol_adaln_linear launch");
}

sol_status sol_adaln_linear_swiglu(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                   const void* shift, const void* scale, int64_t ld_mod,
                                   sol_modsel sel, const void* w, int64_t ld_w, void* workspace,
                                   size_t workspace_bytes, int32_t strategy, int64_t n_tokens,
                                   int64_t inner, int64_t d, float eps, sol_dtype dt, sol_stream_t stream)
{
    TRY(check_strategy(strategy));
    const int64_t n_out = 2 * inner;
    TRY(check_linear_shape(n_tokens, n_out, d, dt, 256));
    TRY(check_modsel(sel));
    CHECK(std::isfinite(eps) && eps >= 0.f, SOL_ERR_INVALID_ARGUMENT, "eps must be finite and >= 0");
    TRY(check_tensor("w", w, ld_w, d, dt, true));
    TRY(check_tensor("shift", shift, ld_mod, d, dt, false));
    TRY(check_tensor("scale", scale, ld_mod, d, dt, false));
    if (n_tokens == 0) return SOL_OK;
    AdalnWorkspace lay;
    int64_t R = 0;
    TRY(check_workspace(workspace, workspace_bytes, n_tokens, n_out, d, sel, &lay, &R));
    TRY(check_tensor("out", out, ld_out, inner, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    CHECK(!spans_overlap(out, n_tokens, ld_out, inner, 2, x, n_tokens, ld_x, d, 2) &&
              !spans_overlap(out, n_tokens, ld_out, inner, 2, w, n_out, ld_w, d, 2) &&
              !spans_overlap(out, n_tokens, ld_out, inner, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(x, n_tokens, ld_x, d, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(w, n_out, ld_w, d, 2, workspace, 1, 0, (int64_t)lay.total, 1),
          SOL_ERR_INVALID_ARGUMENT, "out, x or w overlaps another argument");
    sol::LinearLaunch L = linear_base(out, ld_out, x, ld_x, w, ld_w, n_tokens, n_out, d);
    const sol::ModSel ms = to_dev(sel, n_tokens);
    set_workspace(L, workspace, lay, R);
    L.shift = shift;
    L.scale = scale;
    L.ld_mod = ld_mod;
    L.sel = &ms;
    L.eps = eps;
    L.adaln_strategy = strategy;
    return cuda_status(sol::launch_linear(sol::LINEAR_SWIGLU, true, L, (cudaStream_t)stream),
                       "sol_adaln_linear_swiglu launch");
}

sol_status sol_adaln_qkv_rope(void* qkv, int64_t ld_qkv, const void* x, int64_t ld_x,
                              const void* shift, const void* scale, int64_t ld_mod, sol_modsel sel,
                              const void* w, int64_t ld_w, void* workspace, size_t workspace_bytes,
                              int32_t strategy, const void* wq, const void* wk, const int32_t* pos,
                              int32_t grid_T, int32_t grid_H, int32_t grid_W, const sol_rope3d* rope,
                              int64_t n_tokens, int32_t n_heads, int32_t head_dim, int64_t d, float eps,
                              sol_dtype dt, sol_stream_t stream)
{
    TRY(check_strategy(strategy));
    CHECK(dt == SOL_DTYPE_BF16, SOL_ERR_UNSUPPORTED, "the linear-layer calls take bf16 only");
    CHECK(head_dim == 128, SOL_ERR_UNSUPPORTED, "sol_adaln_qkv_rope is built for head_dim 128 (got %d)",
          (int)head_dim);
    CHECK(n_heads >= 2 && n_heads % 2 == 0, SOL_ERR_UNSUPPORTED,
          "sol_adaln_qkv_rope needs an even n_heads (two heads per 256-column tile), got %d", (int)n_heads);
    TRY(check_modsel(sel));
    TRY(check_qk_common(rope, pos, grid_T, grid_H, grid_W, sel.tokens_per_sample, n_tokens, n_heads, head_dim,
                        eps, dt, wq, wk));
    const int64_t n_out = 3 * (int64_t)n_heads * head_dim;
    TRY(check_linear_shape(n_tokens, n_out, d, dt, 256));
    TRY(check_tensor("w", w, ld_w, d, dt, true));
    TRY(check_tensor("shift", shift, ld_mod, d, dt, false));
    TRY(check_tensor("scale", scale, ld_mod, d, dt, false));
    if (n_tokens == 0) return SOL_OK;
    AdalnWorkspace lay;
    int64_t R = 0;
    TRY(check_workspace(workspace, workspace_bytes, n_tokens, n_out, d, sel, &lay, &R));
    TRY(check_tensor("qkv", qkv, ld_qkv, n_out, dt, true));
    TRY(check_tensor("x", x, ld_x, d, dt, true));
    CHECK(!spans_overlap(qkv, n_tokens, ld_qkv, n_out, 2, x, n_tokens, ld_x, d, 2) &&
              !spans_overlap(qkv, n_tokens, ld_qkv, n_out, 2, w, n_out, ld_w, d, 2) &&
              !spans_overlap(qkv, n_tokens, ld_qkv, n_out, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(x, n_tokens, ld_x, d, 2, workspace, 1, 0, (int64_t)lay.total, 1) &&
              !spans_overlap(w, n_out, ld_w, d, 2, workspace, 1, 0, (int64_t)lay.total, 1),
          SOL_ERR_INVALID_ARGUMENT, "qkv, x or w overlaps another argument");
    sol::LinearLaunch L = linear_base(qkv, ld_qkv, x, ld_x, w, ld_w, n_tokens, n_out, d);
    const sol::ModSel ms = to_dev(sel, n_tokens);
    set_workspace(L, workspace, lay, R);
    L.shift = shift;
    L.scale = scale;
    L.ld_mod = ld_mod;
    L.sel = &ms;
    L.eps = eps;
    L.adaln_strategy = strategy;
    L.wq = wq;
    L.wk = wk;
    L.pos = pos;
    L.grid_H = grid_H;
    L.grid_W = grid_W;
    L.tps = sel.tokens_per_sample;
    L.rope = rope->view;
    L.qk_cols = 2 * n_heads * head_dim;
    return cuda_status(sol::launch_linear(sol::LINEAR_QKROPE, true, L, (cudaStream_t)stream),
                       "sol_adaln_qkv_rope launch");
}

}  // extern "C"
