/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the fused DiT per-token operators.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library (dit_block_b200/) may
 * include, link or call this file; it shares no source with it.  Only tests/,
 * __graft_entry__.smoke() and bench.py's CPU-baseline / reference arm use it.
 *
 * Sources.  The operators are named, but not written out, on two pages:
 *   [XHH-QA]  "8xH200 上的 MiniMax-H3: 无损加速 1.95 倍, SSIM 0.76-0.91 下最高 6.24 倍"
 *             (xhh.club digest of the SGLang Diffusion post), Q&A, the answer on which
 *             operations the fused kernels optimise: AdaLN modulation, the gated
 *             residual, the SwiGLU activation, QK RMSNorm fused with 3D RoPE.
 *   [STM-GAN] "SGLang acelera video do MiniMax-H3 em ate 6,2x em GPUs H200"
 *             (stamatios.com), section "De onde vem os ganhos": AdaLN, SwiGLU,
 *             QK RMSNorm and RoPE kernels.
 *   [STM-RES] same page, section "Resultado principal": the fused kernels cut memory
 *             traffic, intermediate tensors and launches WITHOUT changing the math,
 *             and video and audio tokens share one packed DiT stack.
 * The formulas are the standard definitions of these operators; every point the pages
 * leave open is settled by one stated reading (listed in the repository's design notes):
 *   AdaLN:   h = LN(x) * (1 + scale) + shift, LN without affine, biased variance,
 *            eps inside the square root, two-pass mean then variance.
 *   gated:   o = x + gate * y (gate is a plain multiplier).
 *   SwiGLU:  o_j = silu(a_j) * b_j, silu(v) = v / (1 + e^-v), a = first half, b = second.
 *   QK norm: per head vector, v_i / sqrt(mean(v^2) + eps) * w_i, then 3D RoPE.
 *   3D RoPE: head dims split in chunks (t, h, w) of widths (Dt, Dh, Dw), in that order;
 *            inside chunk c the interleaved pair (2j, 2j+1) turns by
 *            phi = p_c * theta^(-2j / D_c), p_c the token's integer position on axis c.
 *   Modulation row of token n: r = (n / tokens_per_sample) * n_streams + stream_id[n].
 *   Implicit positions (pos == NULL): n_local = n mod tokens_per_sample,
 *            t = n_local / (H*W), h = (n_local / W) mod H, w = n_local mod W.
 *
 * Row subsets: every function takes `rows`, NULL or the global token index of each row
 * passed (row n of the inputs and outputs is token rows[n] of the sequence).  The global
 * index selects the modulation row, the stream id (stream_id and pos are indexed by it)
 * and the implicit grid position; it lets a caller check sampled rows of a long
 * sequence without handing over the whole sequence.
 *
 * Every input element is read through load(), which widens f32 / bf16 / f64 to double
 * exactly.  Everything after that is fp64; nothing is rounded until the caller reads
 * the fp64 output.  Rows run in parallel with OpenMP; nothing else is reordered.
 *
 * Parity pins: every function here is pinned by tests/test_oracle_pins.py (library
 * special cases, invariants, closed forms and brute force on tiny inputs).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_BF16 = 1, OR_F64 = 2 };

/* Widen one stored element to double.  bf16 is the upper half of an IEEE binary32,
 * so shifting its 16 bits left by 16 gives the binary32 with the same value. */
static double load(const void* base, int dt, int64_t idx)
{
    if (dt == OR_F64) return ((const double*)base)[idx];
    if (dt == OR_F32) return (double)((const float*)base)[idx];
    uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Modulation row for token n [STM-RES: one packed stack for video and audio, so each
 * token picks the shift/scale/gate row of its own sample and stream]. */
static int64_t mod_row(int64_t n, const uint8_t* stream_id, int32_t n_streams,
                       int64_t tokens_per_sample)
{
    int64_t sample = tokens_per_sample > 0 ? n / tokens_per_sample : 0;
    int64_t stream = stream_id ? (int64_t)stream_id[n] : 0;
    return sample * (int64_t)n_streams + stream;
}

/* AdaLN modulation [XHH-QA, STM-GAN]:
 *   mu = mean(x), var = mean((x - mu)^2), h = (x - mu)/sqrt(var + eps)*(1 + scale) + shift.
 * shift or scale NULL means a zero vector. */
void oracle_adaln_modulate(double* h, int64_t ld_h,
                           const void* x, int64_t ld_x, int dt_x,
                           const void* shift, const void* scale, int64_t ld_mod, int dt_mod,
                           const uint8_t* stream_id, int32_t n_streams, int64_t tokens_per_sample,
                           const int64_t* rows, int64_t n_tokens, int64_t d, double eps)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        const int64_t r = mod_row(rows ? rows[n] : n, stream_id, n_streams, tokens_per_sample);
        double mu = 0.0;
        for (int64_t i = 0; i < d; ++i) mu += load(x, dt_x, n * ld_x + i);
        mu /= (double)d;
        double var = 0.0;
        for (int64_t i = 0; i < d; ++i) {
            const double c = load(x, dt_x, n * ld_x + i) - mu;
            var += c * c;
        }
        var /= (double)d;
        const double rstd = 1.0 / sqrt(var + eps);
        for (int64_t i = 0; i < d; ++i) {
            const double sc = scale ? load(scale, dt_mod, r * ld_mod + i) : 0.0;
            const double sh = shift ? load(shift, dt_mod, r * ld_mod + i) : 0.0;
            const double xn = (load(x, dt_x, n * ld_x + i) - mu) * rstd;
            h[n * ld_h + i] = xn * (1.0 + sc) + sh;
        }
    }
}

/* Gated residual [XHH-QA]: o = x + gate * y.  gate NULL means zero. */
void oracle_gated_residual(double* o, int64_t ld_o,
                           const void* x, int64_t ld_x, const void* y, int64_t ld_y, int dt_xy,
                           const void* gate, int64_t ld_mod, int dt_mod,
                           const uint8_t* stream_id, int32_t n_streams, int64_t tokens_per_sample,
                           const int64_t* rows, int64_t n_tokens, int64_t d)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        const int64_t r = mod_row(rows ? rows[n] : n, stream_id, n_streams, tokens_per_sample);
        for (int64_t i = 0; i < d; ++i) {
            const double g = gate ? load(gate, dt_mod, r * ld_mod + i) : 0.0;
            o[n * ld_o + i] = load(x, dt_xy, n * ld_x + i) + g * load(y, dt_xy, n * ld_y + i);
        }
    }
}

/* Gated residual with the Cache-DiT residual-change statistics [XHH-QA, the answer on
 * how Cache-DiT reuses computation: after warm-up steps it compares the normalised
 * residual change of boundary blocks with the cached state and reuses the cache when
 * the change is below a threshold].  Read here as: the block's residual contribution
 * r = gate * y, compared with the cached r of the previous step, per sample:
 *     sums[s][0] = sum |r - cache|,   sums[s][1] = sum |cache|
 * over every element of the sample's tokens (video and audio together: one joint
 * decision for the packed stack [STM-RES]); the change is sums[s][0] / sums[s][1].
 * out = x + r as in oracle_gated_residual; r_out receives r (the refreshed cache).
 * sums must hold 2 * n_samples doubles and is overwritten. */
void oracle_gated_residual_cache_diff(double* o, double* r_out, double* sums, int64_t n_samples,
                                      const void* x, int64_t ld_x, const void* y, int64_t ld_y,
                                      int dt_xy, const void* gate, int64_t ld_mod, int dt_mod,
                                      const void* cache, int64_t ld_c, int dt_c,
                                      const uint8_t* stream_id, int32_t n_streams,
                                      int64_t tokens_per_sample, const int64_t* rows,
                                      int64_t n_tokens, int64_t d)
{
    for (int64_t s = 0; s < 2 * n_samples; ++s) sums[s] = 0.0;
    for (int64_t n = 0; n < n_tokens; ++n) {
        const int64_t g_n = rows ? rows[n] : n;
        const int64_t r_row = mod_row(g_n, stream_id, n_streams, tokens_per_sample);
        const int64_t sample = tokens_per_sample > 0 ? g_n / tokens_per_sample : 0;
        double dsum = 0.0, csum = 0.0;
        for (int64_t i = 0; i < d; ++i) {
            const double g = gate ? load(gate, dt_mod, r_row * ld_mod + i) : 0.0;
            const double r = g * load(y, dt_xy, n * ld_y + i);
            const double c = load(cache, dt_c, n * ld_c + i);
            o[n * d + i] = load(x, dt_xy, n * ld_x + i) + r;
            r_out[n * d + i] = r;
            dsum += fabs(r - c);
            csum += fabs(c);
        }
        sums[2 * sample] += dsum;
        sums[2 * sample + 1] += csum;
    }
}

/* SwiGLU activation [XHH-QA, STM-GAN]: o_j = a_j / (1 + exp(-a_j)) * b_j.  a and b are
 * separate row pointers so the caller can pass the two halves of one up-projection row
 * (b = a + inner) or two tensors. */
void oracle_swiglu(double* o, int64_t ld_o,
                   const void* a, const void* b, int64_t ld_in, int dt,
                   int64_t n_tokens, int64_t inner)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        for (int64_t j = 0; j < inner; ++j) {
            const double av = load(a, dt, n * ld_in + j);
            const double bv = load(b, dt, n * ld_in + j);
            o[n * ld_o + j] = av / (1.0 + exp(-av)) * bv;
        }
    }
}

/* Position of token n on the three axes (t, h, w). */
static void token_position(int64_t n, const int32_t* pos, int32_t grid_T, int32_t grid_H,
                           int32_t grid_W, int64_t tokens_per_sample, int64_t p[3])
{
    if (pos) {
        p[0] = pos[3 * n + 0];
        p[1] = pos[3 * n + 1];
        p[2] = pos[3 * n + 2];
        return;
    }
    (void)grid_T;
    const int64_t n_local = tokens_per_sample > 0 ? n % tokens_per_sample : n;
    p[0] = n_local / ((int64_t)grid_H * grid_W);
    p[1] = (n_local / grid_W) % grid_H;
    p[2] = n_local % grid_W;
}

/* RMSNorm of one head vector, then 3D RoPE on it [XHH-QA: "QK RMSNorm fused with 3D
 * RoPE"; STM-GAN: QK RMSNorm and RoPE].  in/out are head_dim long; w is the norm weight. */
static void rmsnorm_rope_head(double* out, const void* in, int64_t in_off, int dt,
                              const void* w, int dt_w, int32_t head_dim, double eps,
                              const int64_t p[3], const int32_t dims[3], double theta)
{
    double ms = 0.0;
    for (int32_t i = 0; i < head_dim; ++i) {
        const double v = load(in, dt, in_off + i);
        ms += v * v;
    }
    ms /= (double)head_dim;
    const double inv = 1.0 / sqrt(ms + eps);
    double vn[1024];
    for (int32_t i = 0; i < head_dim; ++i)
        vn[i] = load(in, dt, in_off + i) * inv * (w ? load(w, dt_w, i) : 1.0);

    int32_t off = 0;
    for (int c = 0; c < 3; ++c) {
        const int32_t D = dims[c];
        for (int32_t j = 0; j < D / 2; ++j) {
            const double phi = (double)p[c] * pow(theta, -2.0 * (double)j / (double)D);
            const double cs = cos(phi), sn = sin(phi);
            const double u = vn[off + 2 * j], v = vn[off + 2 * j + 1];
            out[off + 2 * j] = u * cs - v * sn;
            out[off + 2 * j + 1] = u * sn + v * cs;
        }
        off += D;
    }
}

/* QK RMSNorm + 3D RoPE on every head vector of q and of k.  Layout: row n of q starts
 * at n*ld_q and holds n_heads vectors of head_dim; same for k and the two outputs.
 * q or k (with its output) may be NULL to process only the other. Returns 0, or -1 if
 * the split does not fit head_dim. */
int oracle_qk_rmsnorm_rope3d(double* q_out, double* k_out, int64_t ld_qo, int64_t ld_ko,
                             const void* q, const void* k, int64_t ld_q, int64_t ld_k, int dt,
                             const void* wq, const void* wk, int dt_w,
                             const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                             int64_t tokens_per_sample,
                             int32_t dim_t, int32_t dim_h, int32_t dim_w, double theta,
                             const int64_t* rows, int64_t n_tokens, int32_t n_heads,
                             int32_t head_dim, double eps)
{
    const int32_t dims[3] = {dim_t, dim_h, dim_w};
    if (dim_t + dim_h + dim_w != head_dim || (dim_t | dim_h | dim_w) & 1 || head_dim > 1024)
        return -1;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        int64_t p[3];
        token_position(rows ? rows[n] : n, pos, grid_T, grid_H, grid_W, tokens_per_sample, p);
        for (int32_t hh = 0; hh < n_heads; ++hh) {
            if (q)
                rmsnorm_rope_head(q_out + n * ld_qo + (int64_t)hh * head_dim, q,
                                  n * ld_q + (int64_t)hh * head_dim, dt, wq, dt_w, head_dim,
                                  eps, p, dims, theta);
            if (k)
                rmsnorm_rope_head(k_out + n * ld_ko + (int64_t)hh * head_dim, k,
                                  n * ld_k + (int64_t)hh * head_dim, dt, wk, dt_w, head_dim,
                                  eps, p, dims, theta);
        }
    }
    return 0;
}

/* Fused prologue = gated residual then AdaLN on the UNROUNDED residual sum [STM-RES:
 * fusion leaves the math unchanged].  x_out receives x' = x + gate*y (fp64); with
 * y == NULL there is no residual, x' = x and x_out is not written (it may be NULL).
 * x_out and h are dense n_tokens x d. */
void oracle_dit_prologue(double* x_out, double* h,
                         const void* x, const void* y, int dt,
                         const void* gate, const void* shift, const void* scale,
                         int64_t ld, int64_t ld_mod, int dt_mod,
                         const uint8_t* stream_id, int32_t n_streams, int64_t tokens_per_sample,
                         const int64_t* rows, int64_t n_tokens, int64_t d, double eps)
{
    if (y) {
        oracle_gated_residual(x_out, d, x, ld, y, ld, dt, gate, ld_mod, dt_mod, stream_id,
                              n_streams, tokens_per_sample, rows, n_tokens, d);
        oracle_adaln_modulate(h, d, x_out, d, OR_F64, shift, scale, ld_mod, dt_mod, stream_id,
                              n_streams, tokens_per_sample, rows, n_tokens, d, eps);
    } else {
        oracle_adaln_modulate(h, d, x, ld, dt, shift, scale, ld_mod, dt_mod, stream_id,
                              n_streams, tokens_per_sample, rows, n_tokens, d, eps);
    }
}

/* Fused QKV-projection epilogue: QK RMSNorm + 3D RoPE on the q and k slices of packed
 * rows [q | k | v], each n_heads*head_dim wide.  Output rows are [q' | k'] (2*Hh*Dh). */
int oracle_dit_epilogue(double* qk_out, const void* qkv, int64_t ld_qkv, int dt,
                        const void* wq, const void* wk, int dt_w,
                        const int32_t* pos, int32_t grid_T, int32_t grid_H, int32_t grid_W,
                        int64_t tokens_per_sample,
                        int32_t dim_t, int32_t dim_h, int32_t dim_w, double theta,
                        const int64_t* rows, int64_t n_tokens, int32_t n_heads, int32_t head_dim,
                        double eps)
{
    const int64_t hd = (int64_t)n_heads * head_dim;
    const size_t esz = dt == OR_F64 ? 8 : dt == OR_F32 ? 4 : 2;
    const void* k = (const char*)qkv + (size_t)hd * esz;
    return oracle_qk_rmsnorm_rope3d(qk_out, qk_out + hd, 2 * hd, 2 * hd, qkv, k, ld_qkv, ld_qkv,
                                    dt, wq, wk, dt_w, pos, grid_T, grid_H, grid_W,
                                    tokens_per_sample, dim_t, dim_h, dim_w, theta, rows, n_tokens,
                                    n_heads, head_dim, eps);
}

/* Block means for SubBlock routing [XHH-QA on SubBlock sparse attention: the sequence
 * is split into 64-token blocks and a router keeps a fraction of the key blocks;
 * "SGLang acelera video do MiniMax-H3", "De onde vem os ganhos": SubBlock splits the
 * sequence into blocks of 64 tokens].  Read here as: blocks of `block` consecutive
 * tokens that restart at every sample boundary (the last block of a sample holds the
 * remainder); the pooled row of a block is the mean of its tokens' rows of `v`
 * (n_tokens x width, fp64, e.g. the normalised and rotated q or k).  Block b of sample
 * s is row s * ceil(tokens_per_sample / block) + b of `pooled` (width wide).  Returns
 * the number of blocks written. */
int64_t oracle_block_mean(double* pooled, const double* v, int64_t n_tokens, int64_t width,
                          int64_t tokens_per_sample, int64_t block)
{
    const int64_t tps = tokens_per_sample > 0 ? tokens_per_sample : n_tokens;
    const int64_t per_sample = (tps + block - 1) / block;
    int64_t written = 0;
    for (int64_t s0 = 0; s0 < n_tokens; s0 += tps) {
        const int64_t s1 = s0 + tps < n_tokens ? s0 + tps : n_tokens;
        for (int64_t b0 = s0; b0 < s1; b0 += block) {
            const int64_t b1 = b0 + block < s1 ? b0 + block : s1;
            const int64_t row = (s0 / tps) * per_sample + (b0 - s0) / block;
            for (int64_t i = 0; i < width; ++i) {
                double acc = 0.0;
                for (int64_t t = b0; t < b1; ++t) acc += v[t * width + i];
                pooled[row * width + i] = acc / (double)(b1 - b0);
            }
            if (row + 1 > written) written = row + 1;
        }
    }
    return written;
}

/* Convention variants of QK RMSNorm + 3D RoPE (the pages fix neither the norm span nor
 * the rotary pairing; these are the other plausible readings).
 *   norm_span 0: RMS over each head vector, weights [head_dim] (oracle_qk_rmsnorm_rope3d);
 *   norm_span 1: RMS over all n_heads * head_dim elements of the row, weights
 *                [n_heads * head_dim].
 *   pairing 0: interleaved pairs (2j, 2j+1) inside each axis chunk;
 *   pairing 1: rotate-half pairs (j, j + D_c/2) inside each axis chunk, turned by
 *              phi = p_c * theta^(-2j / D_c), j < D_c / 2.
 * Outputs are token-major [n_tokens, n_heads * head_dim]. */
static void norm_rope_row_ex(double* out, const void* in, int64_t in_off, int dt, const void* w,
                             int dt_w, int32_t n_heads, int32_t head_dim, double eps,
                             const int64_t p[3], const int32_t dims[3], double theta,
                             int norm_span, int pairing)
{
    const int64_t hd = (int64_t)n_heads * head_dim;
    double full_inv = 0.0;
    if (norm_span == 1) {
        double ms = 0.0;
        for (int64_t i = 0; i < hd; ++i) {
            const double v = load(in, dt, in_off + i);
            ms += v * v;
        }
        full_inv = 1.0 / sqrt(ms / (double)hd + eps);
    }
    double vn[1024];
    for (int32_t h = 0; h < n_heads; ++h) {
        const int64_t base = (int64_t)h * head_dim;
        double inv = full_inv;
        if (norm_span == 0) {
            double ms = 0.0;
            for (int32_t i = 0; i < head_dim; ++i) {
                const double v = load(in, dt, in_off + base + i);
                ms += v * v;
            }
            inv = 1.0 / sqrt(ms / (double)head_dim + eps);
        }
        for (int32_t i = 0; i < head_dim; ++i) {
            const int64_t wi = norm_span == 1 ? base + i : i;
            vn[i] = load(in, dt, in_off + base + i) * inv * (w ? load(w, dt_w, wi) : 1.0);
        }
        int32_t off = 0;
        for (int c = 0; c < 3; ++c) {
            const int32_t D = dims[c];
            for (int32_t j = 0; j < D / 2; ++j) {
                const double phi = (double)p[c] * pow(theta, -2.0 * (double)j / (double)D);
                const double cs = cos(phi), sn = sin(phi);
                const int32_t a = pairing == 1 ? off + j : off + 2 * j;
                const int32_t b = pairing == 1 ? off + j + D / 2 : off + 2 * j + 1;
                const double u = vn[a], v = vn[b];
                out[base + a] = u * cs - v * sn;
                out[base + b] = u * sn + v * cs;
            }
            off += D;
        }
    }
}

int oracle_qk_rmsnorm_rope3d_ex(double* q_out, double* k_out, const void* q, const void* k,
                                int64_t ld_q, int64_t ld_k, int dt, const void* wq, const void* wk,
                                int dt_w, const int32_t* pos, int32_t grid_T, int32_t grid_H,
                                int32_t grid_W, int64_t tokens_per_sample, int32_t dim_t,
                                int32_t dim_h, int32_t dim_w, double theta, const int64_t* rows,
                                int64_t n_tokens, int32_t n_heads, int32_t head_dim, double eps,
                                int norm_span, int pairing)
{
    const int32_t dims[3] = {dim_t, dim_h, dim_w};
    if (dim_t + dim_h + dim_w != head_dim || (dim_t | dim_h | dim_w) & 1 || head_dim > 1024)
        return -1;
    const int64_t hd = (int64_t)n_heads * head_dim;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tokens; ++n) {
        int64_t p[3];
        token_position(rows ? rows[n] : n, pos, grid_T, grid_H, grid_W, tokens_per_sample, p);
        if (q)
            norm_rope_row_ex(q_out + n * hd, q, n * ld_q, dt, wq, dt_w, n_heads, head_dim, eps, p, dims,
                             theta, norm_span, pairing);
        if (k)
            norm_rope_row_ex(k_out + n * hd, k, n * ld_k, dt, wk, dt_w, n_heads, head_dim, eps, p, dims,
                             theta, norm_span, pairing);
    }
    return 0;
}
