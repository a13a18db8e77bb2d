/*
 * sol.h -- C ABI of libsol, the B200 (sm_100a) library of fused DiT-block per-token
 * operators: AdaLN modulation, the gated residual, the SwiGLU activation, QK RMSNorm
 * fused with 3D RoPE, and two fused chains of them (a block prologue and a QKV
 * epilogue).
 *
 * Sources.  The operators are the ones the SGLang Diffusion write-ups single out as
 * fused kernels for MiniMax-H3:
 *   [XHH-QA]  "8xH200 上的 MiniMax-H3: 无损加速 1.95 倍, SSIM 0.76-0.91 下最高 6.24 倍"
 *             (xhh.club), Q&A, the answer on which operations the fused kernels
 *             optimise: AdaLN modulation, gated residual, SwiGLU activation, and QK
 *             RMSNorm fused with 3D RoPE.
 *   [STM-GAN] "SGLang acelera video do MiniMax-H3 em ate 6,2x em GPUs H200"
 *             (stamatios.com), section "De onde vem os ganhos".
 *   [STM-RES] same page, section "Resultado principal": fused kernels cut memory
 *             traffic, intermediate tensors and launches without changing the math;
 *             video and audio tokens run through one packed DiT stack.
 * The pages name the operators but print no formula; each function below states the
 * formula it computes.
 *
 * Common conventions
 *   Layout.    Token-major: row n of a tensor starts at element n*ld.  Leading
 *              dimensions (ld*) count ELEMENTS and must be multiples of 8 (bf16) or
 *              4 (f32), so that every row starts on a 16-byte boundary.
 *   Pointers.  Device pointers (memory the GPU can address), 16-byte aligned.  The
 *              caller owns every buffer; no op allocates, frees or synchronises.
 *   Dtypes.    All tensors of one call share `dt`.  Arithmetic is fp32 inside every
 *              kernel; each output element is rounded once (round to nearest even)
 *              when stored.  The RoPE tables are always fp32.
 *   Streams.   Every op is asynchronous on `stream` (a cudaStream_t; NULL = the
 *              legacy default stream).  A returned SOL_OK means the launch was
 *              accepted, not that it finished.
 *   Errors.    Arguments are validated on the host before anything is launched; on
 *              failure the call returns a SOL_ERR_* code with no side effect, and
 *              sol_last_error() gives a one-line reason (per host thread).
 *              SOL_ERR_CUDA reports a launch failure.
 *   n_tokens == 0 is valid and launches nothing; tensor pointers may then be NULL.
 *   Aliasing.  Only the aliases each function lists are allowed (every row is read
 *              completely before it is written).  Any other overlap is undefined.
 *   Kernel choice.  Each op picks its kernel from the shape and dtype of the call alone (the
 *              register-resident and streaming kernels where they fit, general ones
 *              otherwise); every choice computes the same values within the stated
 *              tolerance.  Nothing is read from the process environment.
 */
#ifndef SOL_H
#define SOL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st* sol_stream_t; /* same type as cudaStream_t */

typedef enum {
    SOL_OK = 0,
    SOL_ERR_INVALID_ARGUMENT = 1, /* NULL where a tensor is required, bad size or ld  */
    SOL_ERR_MISALIGNED = 2,       /* pointer not 16-byte aligned                        */
    SOL_ERR_UNSUPPORTED = 3,      /* valid but not built: dtype, head_dim, ...           */
    SOL_ERR_CUDA = 4              /* the CUDA runtime refused the launch or allocation */
} sol_status;

typedef enum { SOL_DTYPE_F32 = 0, SOL_DTYPE_BF16 = 1 } sol_dtype;

/* Which modulation row (shift / scale / gate) a token uses.  One packed sequence holds
 * `B` samples of `tokens_per_sample` tokens each; inside a sample each token belongs
 * to one of `n_streams` streams (video, audio, ...) [STM-RES].  Token n uses row
 *     r = (n / tokens_per_sample) * n_streams + stream_id[n]
 * of every modulation tensor, so those tensors hold B*n_streams rows of `ld_mod`.
 *   stream_id          device uint8 [n_tokens], or NULL (every token in stream 0);
 *                      ids >= n_streams are clamped to n_streams - 1.
 *   n_streams          >= 1.
 *   tokens_per_sample  > 0, or 0 meaning the whole call is one sample. */
typedef struct {
    const uint8_t* stream_id;
    int32_t n_streams;
    int64_t tokens_per_sample;
} sol_modsel;

/* Fixed description of a status code (never NULL). */
const char* sol_status_string(sol_status status);

/* One-line reason for the last non-SOL_OK status returned on this host thread ("" if
 * none).  The pointer stays valid until the next sol_* call on this thread. */
const char* sol_last_error(void);

/* Version of this ABI (incremented on any incompatible change). */
int32_t sol_abi_version(void);

/* Error flags raised on the current device by libsol kernels since the last clear:
 * bit 0 = an AdaLN / prologue kernel's bounded wait on its own asynchronous copy gave up;
 * bit 1 = a QK RMSNorm + RoPE kernel's bounded wait on its own asynchronous copy gave up;
 * bit 2 = sol_selftest_wait_timeout's wait gave up (as it is meant to);
 * bits 8..15 = a linear-layer kernel (sol_linear*, sol_adaln_*) gave up a bounded wait
 * in its copy / MMA / epilogue / transform pipeline.  The kernel recorded it, drained
 * its own copies and MMAs, stopped early and left its outputs incomplete.  Synchronises
 * the current device first; clear != 0 resets the flags.  Never set in normal
 * operation. */
sol_status sol_device_errors(uint32_t* flags, int32_t clear);

/* Diagnostic of the failure path above, safe to run at any time: launches one CTA on
 * `stream` that waits, with the same bounded wait the kernels use, on an mbarrier phase
 * that can never complete (it expects two arrivals and gets one); after `polls` polls
 * (1..1000, each suspending for at most about a millisecond) the wait gives up, the CTA
 * records bit 2 of the device error flags and returns.  Nothing faults and the context stays
 * usable: a caller can check that sol_device_errors reports the bit, clear it and go on. */
sol_status sol_selftest_wait_timeout(int32_t polls, sol_stream_t stream);

/* AdaLN modulation [XHH-QA, STM-GAN]:
 *     mu = mean_i x_i,  var = mean_i (x_i - mu)^2  (biased, two passes),
 *     h_i = (x_i - mu) / sqrt(var + eps) * (1 + scale[r]_i) + shift[r]_i
 * for every token row of x (width d); r from `sel`.  LayerNorm has no affine weights:
 * the modulation is its affine part.
 *   h, ld_h        output [n_tokens, ld_h]; may equal x (then ld_h must equal ld_x).
 *   x, ld_x        input  [n_tokens, ld_x].
 *   shift, scale   [rows, ld_mod] or NULL (read as all zero).
 *   d              row width: multiple of 8 (bf16) / 4 (f32), 8 <= d <= 16384.
 *   eps            >= 0, finite. */
sol_status sol_adaln_modulate(void* h, int64_t ld_h, const void* x, int64_t ld_x,
                              const void* shift, const void* scale, int64_t ld_mod,
                              sol_modsel sel, int64_t n_tokens, int64_t d, float eps,
                              sol_dtype dt, sol_stream_t stream);

/* Gated residual [XHH-QA]:  out_i = x_i + gate[r]_i * y_i  (gate is a plain multiplier).
 *   out, ld_out    output [n_tokens, ld_out]; may equal x (then ld_out == ld_x).
 *   x, y           inputs [n_tokens, ld_x] and [n_tokens, ld_y].
 *   gate           [rows, ld_mod] or NULL (zero: out = x, bit for bit, for finite y).
 *   d              multiple of 8 (bf16) / 4 (f32), >= 8. */
sol_status sol_gated_residual(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                              const void* y, int64_t ld_y, const void* gate, int64_t ld_mod,
                              sol_modsel sel, int64_t n_tokens, int64_t d, sol_dtype dt,
                              sol_stream_t stream);

/* Gated residual fused with the Cache-DiT residual-change statistics [XHH-QA, the answer
 * on how Cache-DiT reuses computation between denoising steps: boundary blocks compare
 * the normalised residual change with the cached state; below a threshold the middle
 * blocks reuse the cache, otherwise they recompute and refresh it; STM-RES: one joint
 * decision for the packed video+audio stack].  In one pass over the tokens:
 *     out_i = x_i + gate[r]_i * y_i                  (exactly as sol_gated_residual)
 *     r_i   = gate[r]_i * y_i                        (the block's residual contribution)
 *     sums[s][0] = sum |r_i - cache_i|,  sums[s][1] = sum |cache_i|
 * over every element of every token of sample s (all streams together); the change is
 * sums[s][0] / sums[s][1] and the reuse decision is the caller's.  With refresh != 0
 * the cache is overwritten by r (rounded to dt), so the next step compares against it.
 *   cache, ld_cache  [n_tokens, ld_cache] device tensor, read (and written if refresh);
 *                    must not overlap out, x or y.
 *   sums             device double [n_samples][2], cleared and filled by this call
 *                    (accumulated with fp64 atomics, so the last bits may vary run to
 *                    run); n_samples >= the samples the tokens span.
 * Everything else as in sol_gated_residual. */
sol_status sol_gated_residual_cache_diff(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                         const void* y, int64_t ld_y, const void* gate,
                                         int64_t ld_mod, sol_modsel sel, void* cache,
                                         int64_t ld_cache, int32_t refresh, double* sums,
                                         int64_t n_samples, int64_t n_tokens, int64_t d,
                                         sol_dtype dt, sol_stream_t stream);

/* SwiGLU activation [XHH-QA, STM-GAN]:  out_j = silu(a_j) * b_j,  silu(v) = v/(1+e^-v),
 * j < inner, for every token row.  For the packed up-projection u = [a | b] of width
 * 2*inner pass a = u, b = u + inner (elements) and ld_in = ld of u.
 *   out, ld_out    output [n_tokens, ld_out], must not overlap a or b.
 *   a, b, ld_in    inputs; row n of a (b) starts at a + n*ld_in (b + n*ld_in).
 *   inner          multiple of 8 (bf16) / 4 (f32), >= 8. */
sol_status sol_swiglu(void* out, int64_t ld_out, const void* a, const void* b, int64_t ld_in,
                      int64_t n_tokens, int64_t inner, sol_dtype dt, sol_stream_t stream);

/* 3D RoPE tables (library-owned).  The head vector is split into three chunks of widths
 * dim_t, dim_h, dim_w (in this order, each even, summing to head_dim).  Inside chunk c,
 * the interleaved pair (2j, 2j+1) of a token at integer position p_c on axis c turns by
 *     phi = p_c * theta^(-2j / dim_c).
 * The tables hold cos(phi), sin(phi) for p_c in [0, max_c), computed on the host in fp64
 * and rounded to fp32.  Create allocates device memory on the CURRENT device (one
 * cudaMalloc, one synchronous copy); use the handle only on that device.  Destroy
 * frees it (NULL is accepted) and must not run while a kernel using it is in flight. */
typedef struct sol_rope3d sol_rope3d;
sol_status sol_rope3d_create(sol_rope3d** out, int32_t dim_t, int32_t dim_h, int32_t dim_w,
                             double theta, int32_t max_t, int32_t max_h, int32_t max_w);
sol_status sol_rope3d_destroy(sol_rope3d* rope);

/* QK RMSNorm fused with 3D RoPE [XHH-QA "QK RMSNorm 与 3D RoPE 的融合", STM-GAN]:
 * for every head vector v (head_dim wide) of q and of k:
 *     v^_i = v_i / sqrt(mean_i v_i^2 + eps) * w_i         (w = wq for q, wk for k)
 * then every pair of v^ is turned by the RoPE angle of the token's (t, h, w) position.
 *   q_out, k_out   outputs, ld_qo / ld_ko; may equal q / k (in place) with the same ld.
 *   q, k           [n_tokens, ld_q] / [n_tokens, ld_k]: n_heads vectors per row, the
 *                  row may sit inside a packed QKV row (ld = 3*n_heads*head_dim).
 *   wq, wk         [head_dim] RMSNorm weights, or NULL (all ones).
 *   pos            device int32 [n_tokens, 3] (t, h, w) positions, or NULL: then token
 *                  n of each sample sits at n_local = n mod tokens_per_sample in a
 *                  row-major grid_T x grid_H x grid_W grid:
 *                  t = n_local / (H*W), h = (n_local / W) mod H, w = n_local mod W.
 *                  Explicit positions outside [0, max_c) are clamped into it.
 *   grid_*         used when pos == NULL; each must be <= the table's max on its axis.
 *   tokens_per_sample  > 0, or 0 = one sample (used only when pos == NULL).
 *   rope           tables from sol_rope3d_create, dims summing to head_dim.
 *   head_dim       64, 128 or 256 for bf16; 32, 64 or 128 for f32.
 *   n_heads        >= 1. */
sol_status sol_qk_rmsnorm_rope3d(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko,
                                 const void* q, const void* k, int64_t ld_q, int64_t ld_k,
                                 const void* wq, const void* wk, const int32_t* pos,
                                 int32_t grid_T, int32_t grid_H, int32_t grid_W,
                                 int64_t tokens_per_sample, const sol_rope3d* rope,
                                 int64_t n_tokens, int32_t n_heads, int32_t head_dim,
                                 float eps, sol_dtype dt, sol_stream_t stream);

/* QK RMSNorm + 3D RoPE in the other conventions the pages leave open, and with outputs
 * at any (token, head, sample) strides -- e.g. straight into an attention-friendly
 * [sample, head, token, dim] layout.
 *   norm_span     SOL_NORM_PER_HEAD: RMS over each head vector, weights [head_dim] (as
 *                 sol_qk_rmsnorm_rope3d);  SOL_NORM_ACROSS_HEADS: RMS over all
 *                 n_heads * head_dim elements of the row, weights [n_heads * head_dim].
 *   rope_pairing  SOL_ROPE_INTERLEAVED: pairs (2j, 2j+1) inside each axis chunk (as
 *                 sol_qk_rmsnorm_rope3d);  SOL_ROPE_HALF: pairs (j, j + D_c/2), angle
 *                 p_c * theta^(-2j/D_c); needs every chunk width to be a multiple of 16
 *                 (bf16) or 8 (f32).
 *   Outputs       element (token n, head h, dim i) of q (k) goes to
 *                     q_out[s * out_sample_stride + (n - s * tokens_per_sample) * out_token_stride
 *                           + h * out_head_stride + i],   s = n / tokens_per_sample
 *                 (s = 0 when tokens_per_sample is 0).  Strides are in elements, multiples
 *                 of 8 (bf16) / 4 (f32).  Token-major rows: token = ld, head = head_dim,
 *                 sample = tokens_per_sample * ld.  Head-major [S, H, N, D]: token =
 *                 head_dim, head = N * head_dim, sample = H * N * head_dim.  An output may
 *                 equal its input only with the input's own token-major strides; otherwise
 *                 outputs must not overlap the inputs.
 *   Other fields as in sol_qk_rmsnorm_rope3d. */
typedef enum { SOL_NORM_PER_HEAD = 0, SOL_NORM_ACROSS_HEADS = 1 } sol_norm_span;
typedef enum { SOL_ROPE_INTERLEAVED = 0, SOL_ROPE_HALF = 1 } sol_rope_pairing;
typedef struct {
    void* q_out;
    void* k_out;
    int64_t out_token_stride, out_head_stride, out_sample_stride;
    const void* q;
    const void* k;
    int64_t ld_q, ld_k;
    const void* wq;
    const void* wk;
    const int32_t* pos;
    int32_t grid_T, grid_H, grid_W;
    int64_t tokens_per_sample;
    const sol_rope3d* rope;
    int64_t n_tokens;
    int32_t n_heads, head_dim;
    float eps;
    int32_t norm_span;    /* sol_norm_span */
    int32_t rope_pairing; /* sol_rope_pairing */
    sol_dtype dt;
} sol_qk_desc;
sol_status sol_qk_rmsnorm_rope3d_ex(const sol_qk_desc* desc, sol_stream_t stream);

/* Fused block prologue [STM-RES: one pass instead of two, same math]:
 *     x'_i = x_i + gate[r]_i * y_i             (skipped when y == NULL: x' = x)
 *     h_i  = AdaLN(x')_i  as in sol_adaln_modulate, on the UNROUNDED fp32 x'.
 * One read of x (and y), one write of x' (when y != NULL) and of h.
 *   x_out          [n_tokens, ld] receives x' (rounded); required iff y != NULL; may
 *                  equal x.
 *   h              [n_tokens, ld]; must not overlap x, y or x_out.
 *   gate, shift, scale  [rows, ld_mod] or NULL (zero).
 *   ld             shared leading dimension of x_out, h, x, y. */
sol_status sol_dit_prologue(void* x_out, void* h, const void* x, const void* y,
                            const void* gate, const void* shift, const void* scale, int64_t ld,
                            int64_t ld_mod, sol_modsel sel, int64_t n_tokens, int64_t d,
                            float eps, sol_dtype dt, sol_stream_t stream);

/* Fused QKV-projection epilogue: sol_qk_rmsnorm_rope3d on the q and k parts of packed
 * rows [q | k | v] (q at element 0, k at n_heads*head_dim), IN PLACE, in one launch;
 * v is neither read nor written.  Arguments as in sol_qk_rmsnorm_rope3d. */
sol_status sol_dit_epilogue(void* qkv, int64_t ld_qkv, const void* wq, const void* wk,
                            const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                            int64_t tokens_per_sample, const sol_rope3d* rope, int64_t n_tokens,
                            int32_t n_heads, int32_t head_dim, float eps, sol_dtype dt,
                            sol_stream_t stream);

/* Number of SubBlock blocks of `block_tokens` tokens in a packed sequence: blocks
 * restart at every sample boundary, so it is n_samples * ceil(tokens_per_sample /
 * block_tokens) (tokens_per_sample 0 = one sample); 0 for invalid arguments. */
int64_t sol_subblock_count(int64_t n_tokens, int64_t tokens_per_sample, int32_t block_tokens);

/* The QKV epilogue fused with the block means SubBlock sparse attention routes on
 * [XHH-QA, the answer on SubBlock: 64-token blocks, a router keeps a fraction of the key
 * blocks; STM-GAN, SubBlock splits the sequence into blocks of 64 tokens].  Does exactly
 * what sol_dit_epilogue does (q and k of packed [q | k | v] rows normalised and rotated
 * in place) and, in the same pass, writes the mean of the resulting q (k) rows of every
 * block into pooled_q (pooled_k): block b of sample s is row
 * s * ceil(tokens_per_sample / block_tokens) + b; the last block of a sample averages
 * the tokens it has.  Means are taken over the fp32 results before their rounding.
 *   pooled_q, pooled_k  [sol_subblock_count(...), ld_pool] each; must not overlap
 *                       each other or qkv.
 *   block_tokens        tokens per block (64 on the pages), >= 1.
 * Other arguments as in sol_dit_epilogue; the per-block fp32 accumulator,
 * 2 * n_heads * (head_dim + 16) floats, must fit 110 KiB (head_dim 128: up to 95 heads). */
sol_status sol_dit_epilogue_pool(void* qkv, int64_t ld_qkv, const void* wq, const void* wk,
                                 const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                                 int64_t tokens_per_sample, const sol_rope3d* rope, int64_t n_tokens,
                                 int32_t n_heads, int32_t head_dim, float eps, void* pooled_q,
                                 void* pooled_k, int64_t ld_pool, int32_t block_tokens, sol_dtype dt,
                                 sol_stream_t stream);

/* One pass of the block's per-token hot path over HOST-resident tensors [STM-RES: the
 * fused operators cut memory traffic and per-step launches; video and audio tokens run
 * through one packed DiT stack].  Computes exactly what these five device calls compute
 * over the whole sequence, in this order:
 *     h1      = sol_adaln_modulate(x; shift_msa, scale_msa)
 *     q|k     = sol_dit_epilogue(qkv)                    (in place on the qkv rows)
 *     x1, h2  = sol_dit_prologue(x, y_attn; gate_msa, shift_mlp, scale_mlp)
 *     act     = sol_swiglu(u)                            (u = [a | b], inner wide)
 *     x2      = sol_gated_residual(x1, y_mlp; gate_mlp)
 * but with every token-row tensor in host memory: the sequence is cut into chunks of at
 * most `chunk_tokens` tokens that never cross a sample, and each chunk is copied in
 * (cudaMemcpyAsync on s_in), computed (the five launches on s_comp) and copied out
 * (on s_out) through `n_slots` rotating device buffers in the caller's workspace, so that
 * the copies of neighbouring chunks overlap the compute.  Inputs and outputs should be
 * page-locked (cudaHostAlloc / cudaHostRegister) for the copies to run asynchronously.
 *
 * Ordering: s_in and s_out first wait for the work already enqueued on s_comp; when the
 * call returns, s_comp has been made to wait for the last copy-out, so anything enqueued
 * on s_comp afterwards (a cudaStreamSynchronize, an event) sees the complete pass and
 * the host outputs filled.  The three streams must be distinct.  The call itself does not
 * block the host (except where the copies are from pageable memory).
 *
 * Host tensors (token-major, rows contiguous: ld = row width):
 *   x, y_attn, y_mlp   [n_tokens, d]          required
 *   qkv                [n_tokens, 3 * hd]     required; hd = n_heads * head_dim; q | k | v
 *   u                  [n_tokens, 2 * inner]  required
 *   pos                int32 [n_tokens, 3] or NULL: then each sample's tokens sit on the
 *                      row-major grid_T x grid_H x grid_W grid (as sol_qk_rmsnorm_rope3d)
 *   stream_id          uint8 [n_tokens] or NULL (every token in stream 0)
 *   h1, x1, h2, x2     [n_tokens, d]          outputs; NULL = not copied back
 *   qk                 [n_tokens, 2 * hd]     output: the normalised, rotated q | k; or NULL
 *   act                [n_tokens, inner]      output, or NULL
 *   shift_msa, scale_msa, gate_msa, shift_mlp, scale_mlp, gate_mlp
 *                      [n_samples * n_streams, d] modulation rows (row r = sample *
 *                      n_streams + stream, as sol_modsel), or NULL (zero); n_samples =
 *                      ceil(n_tokens / tokens_per_sample), 1 when tokens_per_sample is 0
 *   wq, wk             [head_dim] RMSNorm weights, or NULL (ones)
 * The modulation rows and weights are copied once per call (on s_in, ahead of the first
 * chunk) into the workspace; rope is the device-side table handle of sol_rope3d_create.
 * Sizes: n_tokens >= 0; tokens_per_sample > 0, or 0 = one sample; n_streams >= 1; d,
 * n_heads, head_dim, inner as the five device calls accept them; eps >= 0.
 * workspace: caller-owned device memory of at least
 * sol_dit_block_host_workspace_bytes(desc, chunk_tokens, n_slots) bytes, 256-byte aligned;
 * chunk_tokens >= 1, n_slots >= 1 (2 or more overlap copies with compute).  The pass uses
 * the workspace until s_comp reaches the end of the pass.
 * Errors: every argument is validated before anything is enqueued; a copy or launch that
 * the CUDA runtime refuses part-way returns SOL_ERR_CUDA and leaves the pass incomplete
 * (what was enqueued stays enqueued). */
typedef struct {
    const void* x;
    const void* qkv;
    const void* y_attn;
    const void* u;
    const void* y_mlp;
    const int32_t* pos;
    const uint8_t* stream_id;
    void* h1;
    void* qk;
    void* x1;
    void* h2;
    void* act;
    void* x2;
    const void* shift_msa;
    const void* scale_msa;
    const void* gate_msa;
    const void* shift_mlp;
    const void* scale_mlp;
    const void* gate_mlp;
    const void* wq;
    const void* wk;
    const sol_rope3d* rope;
    int32_t grid_T, grid_H, grid_W;
    int64_t n_tokens;
    int64_t tokens_per_sample;
    int32_t n_streams;
    int64_t d;
    int32_t n_heads, head_dim;
    int64_t inner;
    float eps;
    sol_dtype dt;
} sol_block_host_desc;

/* Device workspace, in bytes, that sol_dit_block_host needs (0 for invalid sizes). */
size_t sol_dit_block_host_workspace_bytes(const sol_block_host_desc* desc, int64_t chunk_tokens, int32_t n_slots);

sol_status sol_dit_block_host(const sol_block_host_desc* desc, void* workspace, size_t workspace_bytes,
                              int64_t chunk_tokens, int32_t n_slots, sol_stream_t s_in, sol_stream_t s_comp,
                              sol_stream_t s_out);

/* QK RMSNorm + 3D RoPE for callers that cannot allocate device memory.  The pages have
 * no counterpart: this entry point exists for hosts that reserve device memory up front
 * and forbid allocation while they run work (inference engines whose pool already holds
 * nearly all of HBM, plugin execute callbacks, latency-critical loops that cannot afford
 * cudaMalloc's device synchronisation).  sol_qk_rmsnorm_rope3d needs a sol_rope3d handle,
 * and creating one calls cudaMalloc; this function allocates nothing.
 *
 * It computes exactly what sol_qk_rmsnorm_rope3d computes, with the table described by
 * (dim_t, dim_h, dim_w, theta, max_t, max_h, max_w) as in sol_rope3d_create.  The table
 * is rebuilt on `stream` by every call inside a fixed device array of
 * SOL_NOALLOC_MAX_ROPE_ENTRIES (cos, sin) pairs (512 KiB, held by every GPU that loads
 * the library until the process exits); a table needing more entries,
 * max_t*dim_t/2 + max_h*dim_h/2 + max_w*dim_w/2, is rejected with SOL_ERR_UNSUPPORTED.
 * All calls share that array: calls whose kernels overlap on the GPU (other streams,
 * unordered host threads) race on it and must be serialised by the caller.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * current device) and keeps it for the life of the process; make that first call before
 * any stream capture.  The kept address does not survive the device's context: after
 * cudaDeviceReset (or anything else that destroys the primary context) this entry point
 * must not be called again in the process.
 * Other arguments, layouts, aliasing and errors as in sol_qk_rmsnorm_rope3d. */
#define SOL_NOALLOC_MAX_ROPE_ENTRIES 65536
sol_status sol_qk_rmsnorm_rope3d_noalloc(void* q_out, void* k_out, int64_t ld_qo, int64_t ld_ko,
                                         const void* q, const void* k, int64_t ld_q, int64_t ld_k,
                                         const void* wq, const void* wk, const int32_t* pos,
                                         int32_t grid_T, int32_t grid_H, int32_t grid_W,
                                         int64_t tokens_per_sample, int32_t dim_t, int32_t dim_h,
                                         int32_t dim_w, double theta, int32_t max_t,
                                         int32_t max_h, int32_t max_w, int64_t n_tokens,
                                         int32_t n_heads, int32_t head_dim, float eps,
                                         sol_dtype dt, sol_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Linear layers with the per-token operators fused in.
 *
 * [STM-RES] credits the fused kernels with cutting memory traffic, intermediate
 * tensors and launches without changing the math.  In the DiT block the per-token
 * operators sit around its linear layers: AdaLN feeds the QKV projection and QK
 * RMSNorm + 3D RoPE follows it; the gated residual follows the attention output
 * projection and the MLP down projection; SwiGLU follows the MLP up projection.  The
 * calls below run each linear layer on the tensor cores and apply the operator to the
 * operand tile on its way in or to the accumulator on its way out, so the operator's
 * input or output never makes its own trip through HBM.
 *
 * Common rules (in addition to the conventions at the top of this file):
 *   dt must be SOL_DTYPE_BF16 (the tensor cores take bf16 operands; SOL_ERR_UNSUPPORTED
 *   otherwise).  W is [n_out, k] with row stride ld_w: the usual linear-layer layout,
 *   y = a . W^T, no bias.  k must be a multiple of 64 and n_out a multiple of 256
 *   (SOL_ERR_UNSUPPORTED otherwise); n_tokens < 2^31.  The tensor cores read bf16
 *   operands and accumulate in fp32; every output element is rounded once, when
 *   stored.  No output may overlap an input
 *   except where stated.  Each call launches one kernel (the sol_adaln_* calls three:
 *   row statistics, the weight fold, then the linear layer).
 * ------------------------------------------------------------------------------------ */

/* out = a . W^T: a [n_tokens, k], W [n_out, k], out [n_tokens, n_out]. */
sol_status sol_linear(void* out, int64_t ld_out, const void* a, int64_t ld_a, const void* w,
                      int64_t ld_w, int64_t n_tokens, int64_t n_out, int64_t k, sol_dtype dt,
                      sol_stream_t stream);

/* Output / down projection with the gated residual in its epilogue:
 *     out = x + gate[r] * (a . W^T)
 * a [n_tokens, k], W [d, k], x and out [n_tokens, d]; gate [B*n_streams, ld_mod] chosen
 * per token by `sel` as in sol_gated_residual (NULL = zero: out = x).  The product is
 * not rounded before the residual.  out may be x (same pointer and ld). */
sol_status sol_linear_gated_residual(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                     const void* a, int64_t ld_a, const void* w, int64_t ld_w,
                                     const void* gate, int64_t ld_mod, sol_modsel sel,
                                     int64_t n_tokens, int64_t d, int64_t k, sol_dtype dt,
                                     sol_stream_t stream);

/* MLP up projection with SwiGLU in its epilogue:
 *     out[:, j] = silu((a . W1^T)[:, j]) * (a . W2^T)[:, j],   W = [W1; W2]
 * W [2*inner, k] holds the gated half W1 in rows [0, inner) and the multiplying half W2
 * in rows [inner, 2*inner) (the two halves of the packed up projection, in the order
 * sol_swiglu takes them); out [n_tokens, inner]; inner a multiple of 128.  Neither
 * half is rounded before the product. */
sol_status sol_linear_swiglu(void* out, int64_t ld_out, const void* a, int64_t ld_a, const void* w,
                             int64_t ld_w, int64_t n_tokens, int64_t inner, int64_t k, sol_dtype dt,
                             sol_stream_t stream);

/* Device workspace, in bytes, that sol_adaln_linear, sol_adaln_linear_swiglu and
 * sol_adaln_qkv_rope need for n_tokens tokens, n_out output columns and d input columns,
 * with the modulation rows `sel` implies (R = ceil(n_tokens / tokens_per_sample) *
 * n_streams, or n_streams when tokens_per_sample is 0): per token 8 bytes of row
 * statistics, per 128 tokens 4 bytes of modulation-row sets, per modulation row two fp32
 * vectors of n_out, and one region of the larger of the staged h (n_tokens * d bf16) and
 * the folded weights (R * n_out * d bf16).  Returns 0 for invalid sizes or R > 32. */
size_t sol_adaln_workspace_bytes(int64_t n_tokens, int64_t n_out, int64_t d, sol_modsel sel);

/* How the sol_adaln_* calls apply AdaLN in front of their linear layer; every strategy
 * computes the same product within the bf16 bound stated at the top of this section.
 *   SOL_ADALN_STAGE (the fastest on B200): h is written once, rounded to bf16, into the
 *     workspace by the AdaLN row kernel and read back by the GEMM, whose epilogue applies
 *     the fused operator (the per-token operator's output never goes to HBM);
 *   SOL_ADALN_FOLD: h is never formed -- per modulation row r the call writes V_r =
 *     bf16(W * (1 + scale_r)) (column-wise), c_r = sum_k V_r[:, k] and b_r = shift_r . W^T
 *     into the workspace, computes mean and 1/sqrt(var + eps) of every row of x, and runs
 *     one GEMM of x against V_r whose epilogue forms rstd * (acc - mean * c_r) + b_r (the
 *     only rounding of an operand is that of the folded weights, of the same size as
 *     rounding h); a tile whose rows use several modulation rows is computed once per row
 *     used;
 *   SOL_ADALN_TRANSFORM: h is never stored -- each x tile is rewritten as bf16 h in
 *     shared memory before the tensor cores read it. */
typedef enum { SOL_ADALN_STAGE = 0, SOL_ADALN_FOLD = 1, SOL_ADALN_TRANSFORM = 2 } sol_adaln_strategy;

/* AdaLN fused into a linear layer:
 *     out = h . W^T,   h = LN(x) * (1 + scale[r]) + shift[r]   (as sol_adaln_modulate)
 * x [n_tokens, d], W [n_out, d], out [n_tokens, n_out]; d a multiple of 64; at most 32
 * modulation rows (SOL_ERR_UNSUPPORTED otherwise).
 *   strategy       a sol_adaln_strategy (SOL_ERR_INVALID_ARGUMENT otherwise).
 *   workspace      caller-owned device memory of at least sol_adaln_workspace_bytes(...)
 *                  bytes, 256-byte aligned, overlapping no other argument; its contents
 *                  are scratch. */
sol_status sol_adaln_linear(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                            const void* shift, const void* scale, int64_t ld_mod, sol_modsel sel,
                            const void* w, int64_t ld_w, void* workspace, size_t workspace_bytes,
                            int32_t strategy, int64_t n_tokens, int64_t n_out, int64_t d, float eps,
                            sol_dtype dt, sol_stream_t stream);

/* The MLP input of a block in one pass: AdaLN into the up projection, SwiGLU in its
 * epilogue:
 *     out[:, j] = silu((h . W1^T)[:, j]) * (h . W2^T)[:, j],   W = [W1; W2],
 *     h = LN(x) * (1 + scale[r]) + shift[r]   (as sol_adaln_linear)
 * x [n_tokens, d], W [2*inner, d] (gated half first, as sol_linear_swiglu), out
 * [n_tokens, inner]; inner a multiple of 128; workspace and strategy as in
 * sol_adaln_linear with n_out = 2 * inner.  The projection is neither stored nor rounded
 * before the SwiGLU. */
sol_status sol_adaln_linear_swiglu(void* out, int64_t ld_out, const void* x, int64_t ld_x,
                                   const void* shift, const void* scale, int64_t ld_mod,
                                   sol_modsel sel, const void* w, int64_t ld_w, void* workspace,
                                   size_t workspace_bytes, int32_t strategy, int64_t n_tokens,
                                   int64_t inner, int64_t d, float eps, sol_dtype dt,
                                   sol_stream_t stream);

/* The attention input of a block in one pass: AdaLN into the QKV projection, QK RMSNorm
 * + 3D RoPE in its epilogue:
 *     qkv = h . W^T  ([n_tokens, 3*n_heads*head_dim] = q | k | v),  h as in
 *     sol_adaln_linear; then every q and k head vector as sol_dit_epilogue does it
 *     (RMSNorm with wq / wk, interleaved 3D RoPE from `rope`); v as projected.
 * head_dim must be 128 and n_heads even.  Positions: pos [n_tokens, 3] int32, or NULL
 * for the row-major grid (grid_T, grid_H, grid_W) of each sample, samples of
 * sel.tokens_per_sample tokens (0 = one sample), as in sol_qk_rmsnorm_rope3d.
 * workspace and strategy as in sol_adaln_linear (with n_out = 3 * n_heads * head_dim).
 * The projection is not rounded before the norm. */
sol_status sol_adaln_qkv_rope(void* qkv, int64_t ld_qkv, const void* x, int64_t ld_x,
                              const void* shift, const void* scale, int64_t ld_mod, sol_modsel sel,
                              const void* w, int64_t ld_w, void* workspace, size_t workspace_bytes,
                              int32_t strategy, const void* wq, const void* wk, const int32_t* pos,
                              int32_t grid_T, int32_t grid_H, int32_t grid_W, const sol_rope3d* rope,
                              int64_t n_tokens, int32_t n_heads, int32_t head_dim, int64_t d, float eps,
                              sol_dtype dt, sol_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SOL_H */
