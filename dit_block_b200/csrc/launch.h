// launch.h -- host-side launchers of the libsol kernels (internal to the library).
// Arguments reach these only after sol_api.cu validated them.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sol.h"

namespace sol {

struct ModSel;

// Device view of a sol_rope3d: per axis (t, h, w), a [max_c, dim_c/2] table of
// (cos, sin) pairs.
struct RopeDev {
    const float2* tab[3];
    int32_t max[3];
    int32_t half[3];
};

// Element strides of a q/k output: element (token n, head h, dim i) of sample s lives at
// s * sample + (n - s * tokens_per_sample) * token + h * head + i.
struct QkOutStrides {
    int64_t token, head, sample;
};

// Resident CTAs per SM for `kernel` at `block` threads on the current device (cached).
int ctas_per_sm(const void* kernel, int block, size_t smem);
// SM count of the current device (cached).
int sm_count();

cudaError_t launch_gated_residual(sol_dtype dt, void* out, int64_t ld_out, const void* x,
                                  int64_t ld_x, const void* y, int64_t ld_y, const void* gate,
                                  int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                                  cudaStream_t s);

cudaError_t launch_gated_residual_diff(sol_dtype dt, void* out, int64_t ld_out, const void* x,
                                       int64_t ld_x, const void* y, int64_t ld_y, const void* gate,
                                       int64_t ld_mod, void* cache, int64_t ld_c, bool refresh,
                                       double* sums, const ModSel& sel, int64_t n_tokens, int64_t d,
                                       cudaStream_t s);

cudaError_t launch_swiglu(sol_dtype dt, void* out, int64_t ld_out, const void* a, const void* b,
                          int64_t ld_in, int64_t n_tokens, int64_t inner, cudaStream_t s);

// AdaLN with an optional fused gated residual in front (y == nullptr: plain AdaLN).
cudaError_t launch_adaln_rows(sol_dtype dt, void* x_out, int64_t ld_xo, void* h, int64_t ld_h,
                              const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                              const void* gate, const void* shift, const void* scale,
                              int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                              float eps, cudaStream_t s);

cudaError_t launch_qk_rmsnorm_rope3d(sol_dtype dt, void* q_out, void* k_out, int64_t ld_qo,
                                     int64_t ld_ko, const void* q, const void* k, int64_t ld_q,
                                     int64_t ld_k, const void* wq, const void* wk,
                                     const int32_t* pos, int32_t grid_T, int32_t grid_H,
                                     int32_t grid_W, int64_t tokens_per_sample,
                                     const RopeDev& rope, int64_t n_tokens, int32_t n_heads,
                                     int32_t head_dim, float eps, cudaStream_t s);

// QK RMSNorm + 3D RoPE with one warp per (token, q or k) row in registers (k_qk_regs.cu):
// bf16, head_dim 128, an even number of heads; q or k may be NULL.
bool qk_regs_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim);
cudaError_t launch_qk_regs(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                           int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                           int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                           int32_t n_heads, float eps, cudaStream_t s);
// QK RMSNorm + 3D RoPE with one CTA per token, its q and k rows staged in shared memory by
// bulk copies (k_qk_cta.cu): bf16, head_dim 128, an even number of heads up to 48, q and k
// both given.
bool qk_cta_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k, int64_t n_tokens);
cudaError_t launch_qk_cta(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko, const void* q, const void* k,
                          int64_t ld_q, int64_t ld_k, const void* wq, const void* wk, const int32_t* pos,
                          int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope, int64_t n_tokens,
                          int32_t n_heads, float eps, cudaStream_t s);
// The same kernel for the convention variants: norm across heads, rotate-half pairs (chunk
// halves multiples of 4), strided outputs.
bool qk_cta_ex_fits(sol_dtype dt, bool half, int32_t n_heads, int32_t head_dim,
                    const void* q, const void* k, int64_t n_tokens, int64_t tps, const RopeDev& rope);
cudaError_t launch_qk_cta_ex(bool across, bool half, void* q_out, void* k_out, const QkOutStrides& os, const void* q,
                             const void* k, int64_t ld_q, int64_t ld_k, const void* wq, const void* wk,
                             const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps, const RopeDev& rope,
                             int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s);
// The QKV epilogue with block means, staged (k_qk_cta.cu): bf16, head_dim 128, an even
// number of heads up to 48, q and k both given.
bool qk_pool_stage_fits(sol_dtype dt, int32_t n_heads, int32_t head_dim, const void* q, const void* k,
                        int64_t tps, int64_t n_blocks);
cudaError_t launch_qk_pool_stage(void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq, void* pk, int64_t ld_pq,
                                 int64_t ld_pk, const void* wq, const void* wk, const int32_t* pos, int32_t grid_H,
                                 int32_t grid_W, int64_t tps, int32_t block, int64_t bps, int64_t n_blocks,
                                 const RopeDev& rope, int64_t n_tokens, int32_t n_heads, float eps, cudaStream_t s);
// Error flags of these kernels' bounded waits (bit 1); optionally cleared.  Synchronous.
uint32_t qk_device_error(bool clear);

// QK RMSNorm + 3D RoPE, convention variants (k_qk_ex.cu): `across` = RMS over all heads
// with weights [n_heads * head_dim]; `half` = rotate-half pairs; any output strides.
cudaError_t launch_qk_ex(sol_dtype dt, bool across, bool half, void* q_out, void* k_out,
                         const QkOutStrides& os, const void* q, const void* k, int64_t ld_q, int64_t ld_k,
                         const void* wq, const void* wk, const int32_t* pos, int32_t grid_H, int32_t grid_W,
                         int64_t tps, const RopeDev& rope, int64_t n_tokens, int32_t n_heads,
                         int32_t head_dim, float eps, cudaStream_t s);

// QKV epilogue fused with SubBlock block means (k_qk_pool.cu).  In place on q and k.
cudaError_t launch_qk_rope_pool(sol_dtype dt, void* q, void* k, int64_t ld_q, int64_t ld_k, void* pq,
                                void* pk, int64_t ld_pq, int64_t ld_pk, const void* wq, const void* wk,
                                const int32_t* pos, int32_t grid_H, int32_t grid_W, int64_t tps,
                                int32_t block, int64_t bps, int64_t n_blocks, const RopeDev& rope,
                                int64_t n_tokens, int32_t n_heads, int32_t head_dim, float eps,
                                cudaStream_t s);
size_t qk_pool_smem_bytes(sol_dtype dt, int32_t n_heads, int32_t head_dim);
size_t qk_pool_smem_limit();

// Error flags raised on the device by the AdaLN / prologue kernels (bit 0: a bounded
// wait on a bulk copy gave up); optionally cleared.  Synchronous.
uint32_t rows_device_error(bool clear);

// Linear layers on the tensor cores (k_gemm.cu): out = epilogue(A . W^T), bf16 only.
enum LinearEpi { LINEAR_STORE = 0, LINEAR_GATED = 1, LINEAR_SWIGLU = 2, LINEAR_QKROPE = 3 };
struct LinearLaunch {
    int64_t M;          // rows of A (tokens), < 2^31
    int32_t K;          // inner dimension, multiple of 64
    int32_t N;          // rows of W: output columns (SwiGLU: 2 * inner), multiple of 256
    const void* a;      // A [M, K] (row stride ld_a); x for the AdaLN variant
    int64_t ld_a;
    const void* w;      // W [N, K] (row stride ld_w)
    int64_t ld_w;
    void* out;
    int64_t ld_out;
    const void* x;      // gated residual input [M, N]
    int64_t ld_x;
    const void* gate;
    void* stats;        // AdaLN: [M] float2 workspace (mean, rstd)
    const void* shift;
    const void* scale;
    int64_t ld_mod;
    const ModSel* sel;
    const void* wq;     // QK norm weights [128]
    const void* wk;
    const int32_t* pos;
    int32_t grid_H, grid_W;
    int64_t tps;
    RopeDev rope;
    int32_t qk_cols;    // columns of q and k (2 * n_heads * 128)
    float eps;
    // AdaLN folded into the weights (workspace regions)
    uint32_t* rmask;    // [ceil(M / 128)] modulation rows per 128-row block
    void* fold_v;       // workspace region: [n_mod_rows * N, K] bf16 folded weights (fold strategy)
                        // or [M, K] bf16 staged h = AdaLN(x) (stage strategy)
    float* fold_c;      // [n_mod_rows, N]
    float* fold_b;      // [n_mod_rows, N]
    int32_t n_mod_rows; // modulation rows the call may use (<= 32)
    int32_t adaln_strategy;  // sol_adaln_strategy of the sol_adaln_* calls
};
cudaError_t launch_linear(LinearEpi epi, bool adaln, const LinearLaunch& a, cudaStream_t s);
size_t linear_smem_bytes();
// Error flags raised by the linear kernels' bounded waits; optionally cleared.  Synchronous.
uint32_t gemm_device_error(bool clear);

// Store a one-line reason for sol_last_error() on this host thread.
void record_error(const char* msg);

// AdaLN with one warp per row held in registers (k_adaln_warp.cu): whether it takes this
// call, and its launcher.
bool adaln_warp_fits(sol_dtype dt, int64_t d);
cudaError_t launch_adaln_warp(void* h, int64_t ld_h, const void* x, int64_t ld_x, const void* shift,
                              const void* scale, int64_t ld_mod, const ModSel& sel, int64_t n_tokens, int64_t d,
                              float eps, cudaStream_t s);

// Fused prologue with the row in registers (two warps per row, k_adaln_warp.cu).
bool prologue_regs_fits(sol_dtype dt, int64_t d);
cudaError_t launch_prologue_regs(void* x_out, void* h, const void* x, const void* y, const void* gate,
                                 const void* shift, const void* scale, int64_t ld, int64_t ld_mod, const ModSel& sel,
                                 int64_t n_tokens, int64_t d, float eps, cudaStream_t s);

// AdaLN with one CTA per row staged in shared memory by a bulk copy (k_rows_stage.cu): bf16,
// d a multiple of 1024 up to 6144, h and x with one row stride.
bool adaln_stage_fits(sol_dtype dt, int64_t d, int64_t n_tokens);
cudaError_t launch_adaln_stage(void* h, const void* x, int64_t ld, const void* shift, const void* scale, int64_t ld_mod,
                               const ModSel& sel, int64_t n_tokens, int64_t d, float eps, cudaStream_t s);
// Error flags of that kernel's bounded wait (bit 0); optionally cleared.  Synchronous.
uint32_t rows_stage_device_error(bool clear);

// Error flags of sol_selftest_wait_timeout (bit 2); optionally cleared.  Synchronous.
uint32_t selftest_device_error(bool clear);

// Whether a row of `vpr` 16-byte vectors fits the register-resident AdaLN kernel.
bool adaln_row_fits(int64_t vpr);

}  // namespace sol
