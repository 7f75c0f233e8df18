/*
 * Plain fp64 CPU oracle for the per-token hot path of a joint video+audio
 * diffusion-transformer block.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker the CUDA path is
 * compared against.  It is loaded by the tests, by the smoke check and by the
 * CPU-baseline leg of the benchmark, and by nothing else; the product path
 * never calls it.  It shares no code, header, table or helper with the CUDA
 * library: it is written from the definitions below, one row and one element
 * at a time, in double precision, with no blocking, fusion or reordering.
 *
 * Sources of the operations (the pages name the fusions, the textbook
 * definitions they denote fix the arithmetic):
 *   - "fused RMS-AdaLN" and "fused QKNorm + RoPE": Sol Video Inference Engine,
 *     MiniMax-H3 on-device page (nvlabs.github.io/Sana/Sol-Engine/H3-OnDevice),
 *     fusion table ("Fusion | What it eliminates"); the same list appears in
 *     the KOCPC Sol-H3 article, section "Technical Composition: Sol Engine x
 *     Sol-Attn Complete Stack".
 *   - AdaLN branches firing on every denoising step, joint video-plus-audio
 *     single-stream sequence: same H3-OnDevice page, model description; the
 *     ThakiCloud MiniMax-H3 post, section "MiniMax-H3: what the model does,
 *     and how much" (a dense transformer over one joint sequence).
 *   - RMSNorm: y = x / sqrt(mean(x^2) + eps) (Zhang & Sennrich, 2019).
 *   - AdaLN modulation x*(1+scale)+shift and the gated residual h+gate*branch
 *     (adaLN-Zero DiT block, Peebles & Xie, 2023).
 *   - RoPE: pair i of a head rotated by pos * theta^(-2i/d) (Su et al.,
 *     RoFormer, 2021); 3D multimodal split of the frequency list into
 *     t/h/w sections (M-RoPE style), sections 16/24/24 of 64 pairs, theta
 *     10000, audio tokens at positions (t=i,0,0).
 *
 * Readings taken where the pages are silent:
 *   eps inside the square root; mean over all D (or head_dim) channels;
 *   order normalise -> gamma -> modulate; modulation (1 + scale) not scale;
 *   per sample b the rows are the N_v = T*H*W video rows (raster order,
 *   t-major) followed by the audio rows; the modality of row r is video for
 *   r < n_video, audio otherwise; modulation vectors have layout [B, 2, D]
 *   (index 0 video, 1 audio); QKNorm normalises each head over head_dim with
 *   one gamma_q and one gamma_k of length head_dim shared by all heads; the
 *   rotary pair i is the adjacent pair (2i, 2i+1); one frequency index i over
 *   all head_dim/2 pairs, the first sec_t pairs take the t position, the next
 *   sec_h the h position, the last sec_w the w position; rotation is applied
 *   to the normalised, gamma-scaled values with no rounding in between.
 *
 * Inputs are given in the I/O dtype (fp32, or bf16 as raw 16-bit patterns)
 * and are widened exactly to double.  Outputs are unrounded doubles.
 *
 * Row selection: every entry point takes `row_ids`, the global row id
 * (b * L + r) of each of the `n_rows` rows given; the input and output arrays
 * hold just those rows, packed.  row_ids == NULL means rows 0 .. n_rows-1.
 *
 * Every function returns 0 on success and -1 on an argument it cannot use.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* One input element, widened exactly to double. */
static double in_val(const void *base, int64_t i, int dtype)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)base)[i];
    }
    /* bf16 is the upper half of an IEEE binary32 pattern */
    uint32_t bits = (uint32_t)((const uint16_t *)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int64_t row_id(const int64_t *row_ids, int64_t k)
{
    return row_ids ? row_ids[k] : k;
}

/*
 * RMS-AdaLN.  For each given row (sample b, row r in the sample):
 *   ms   = (1/D) * sum_c x[c]^2
 *   n[c] = x[c] / sqrt(ms + eps)
 *   y[c] = n[c] * gamma[c] * (1 + scale[b, m, c]) + shift[b, m, c]
 * with m = 0 (video) if r < n_video else 1 (audio); gamma == NULL means 1.
 * x, y: [n_rows, D]; scale, shift: [B, 2, D]; gamma: [D].
 */
int oracle_rms_adaln(const void *x, const void *scale, const void *shift,
                     const void *gamma, const int64_t *row_ids, int64_t n_rows,
                     int64_t L, int64_t n_video, int64_t D, double eps,
                     int dtype, double *y)
{
    if (n_rows < 0 || L <= 0 || D <= 0 || n_video < 0 || n_video > L)
        return -1;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t g = row_id(row_ids, k);
        int64_t b = g / L;
        int64_t r = g % L;
        int64_t m = (r < n_video) ? 0 : 1;
        int64_t mod = (b * 2 + m) * D; /* offset of this (sample, modality) */

        double ss = 0.0;
        for (int64_t c = 0; c < D; ++c) {
            double v = in_val(x, k * D + c, dtype);
            ss += v * v;
        }
        double ms = ss / (double)D;
        double denom = sqrt(ms + eps);

        for (int64_t c = 0; c < D; ++c) {
            double n = in_val(x, k * D + c, dtype) / denom;
            if (gamma)
                n = n * in_val(gamma, c, dtype);
            double sc = in_val(scale, mod + c, dtype);
            double sh = in_val(shift, mod + c, dtype);
            y[k * D + c] = n * (1.0 + sc) + sh;
        }
    }
    return 0;
}

/*
 * AdaLN-gated residual add.  For each given row (sample b, row r):
 *   out[c] = h[c] + gate[b, m, c] * branch[c],   m as in oracle_rms_adaln.
 * h, branch, out: [n_rows, D]; gate: [B, 2, D].
 */
int oracle_gate_residual(const void *h, const void *branch, const void *gate,
                         const int64_t *row_ids, int64_t n_rows, int64_t L,
                         int64_t n_video, int64_t D, int dtype, double *out)
{
    if (n_rows < 0 || L <= 0 || D <= 0 || n_video < 0 || n_video > L)
        return -1;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t g = row_id(row_ids, k);
        int64_t b = g / L;
        int64_t r = g % L;
        int64_t m = (r < n_video) ? 0 : 1;
        for (int64_t c = 0; c < D; ++c) {
            double hv = in_val(h, k * D + c, dtype);
            double bv = in_val(branch, k * D + c, dtype);
            double gv = in_val(gate, (b * 2 + m) * D + c, dtype);
            out[k * D + c] = hv + gv * bv;
        }
    }
    return 0;
}

/*
 * Gated residual followed by RMS-AdaLN of its result, the chain
 * "h = h + gate1 * attn; x2 = RMS-AdaLN(h)" of the DiT block.  For each
 * given row (sample b, row r, modality m):
 *   hn[c]  = h[c] + gate[b, m, c] * branch[c]          (kept in fp64)
 *   ms     = (1/D) * sum_c hn[c]^2
 *   y[c]   = hn[c] / sqrt(ms + eps) * gamma[c] * (1 + scale[b, m, c])
 *            + shift[b, m, c]
 * Outputs hn (h_out) and y, both [n_rows, D] doubles; the normalisation
 * reads hn unrounded.
 */
int oracle_gate_residual_rms_adaln(const void *h, const void *branch, const void *gate,
                                   const void *scale, const void *shift, const void *gamma,
                                   const int64_t *row_ids, int64_t n_rows, int64_t L,
                                   int64_t n_video, int64_t D, double eps, int dtype,
                                   double *h_out, double *y)
{
    if (n_rows < 0 || L <= 0 || D <= 0 || n_video < 0 || n_video > L)
        return -1;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t g = row_id(row_ids, k);
        int64_t b = g / L;
        int64_t r = g % L;
        int64_t m = (r < n_video) ? 0 : 1;
        int64_t mod = (b * 2 + m) * D;

        double ss = 0.0;
        for (int64_t c = 0; c < D; ++c) {
            double hv = in_val(h, k * D + c, dtype);
            double bv = in_val(branch, k * D + c, dtype);
            double hn = hv + in_val(gate, mod + c, dtype) * bv;
            h_out[k * D + c] = hn;
            ss += hn * hn;
        }
        double denom = sqrt(ss / (double)D + eps);
        for (int64_t c = 0; c < D; ++c) {
            double n = h_out[k * D + c] / denom;
            if (gamma)
                n = n * in_val(gamma, c, dtype);
            y[k * D + c] = n * (1.0 + in_val(scale, mod + c, dtype)) +
                           in_val(shift, mod + c, dtype);
        }
    }
    return 0;
}

/*
 * First-Block-Cache change detector: how far the first block's residual
 * moved since the previous denoising step (the cache gate of the Sol Video
 * Inference Engine MiniMax-H3 page, cross-step caching paragraph: skip the
 * remaining blocks when the first block's residual has barely changed).
 * Relative L1 difference, per sample b over its L*D elements and over the
 * whole batch:
 *   num_b = sum |cur - prev|,  den_b = sum |prev|,
 *   rel_b = num_b / den_b  (0 if num_b == den_b == 0, +inf if only den_b == 0)
 * cur, prev: [B, L, D].  out: [B + 1][3] doubles (num, den, rel), row B for
 * the whole batch (sums of the per-sample num and den).
 */
int oracle_residual_change(const void *cur, const void *prev, int64_t B, int64_t L,
                           int64_t D, int dtype, double *out)
{
    if (B < 0 || L < 0 || D <= 0)
        return -1;
    double tn = 0.0, td = 0.0;
    for (int64_t b = 0; b <= B; ++b) {
        double num = 0.0, den = 0.0;
        if (b < B) {
            for (int64_t i = b * L * D; i < (b + 1) * L * D; ++i) {
                double c = in_val(cur, i, dtype);
                double p = in_val(prev, i, dtype);
                num += fabs(c - p);
                den += fabs(p);
            }
            tn += num;
            td += den;
        } else {
            num = tn;
            den = td;
        }
        out[3 * b + 0] = num;
        out[3 * b + 1] = den;
        out[3 * b + 2] = den > 0.0 ? num / den : (num > 0.0 ? INFINITY : 0.0);
    }
    return 0;
}

/*
 * Position of row r of a sample on the three rotary axes.
 * Video rows r < T*H*W are the latent grid in raster order, t-major:
 *   t = r / (H*W), h = (r / W) mod H, w = r mod W.
 * Audio row i = r - T*H*W sits at (t = i, h = 0, w = 0).
 */
static void row_position(int64_t r, int64_t T, int64_t H, int64_t W,
                         int64_t pos[3])
{
    int64_t n_video = T * H * W;
    if (r < n_video) {
        pos[0] = r / (H * W);
        pos[1] = (r / W) % H;
        pos[2] = r % W;
    } else {
        pos[0] = r - n_video;
        pos[1] = 0;
        pos[2] = 0;
    }
}

/*
 * Per-head QKNorm followed by 3D multimodal RoPE, on the q and k parts of a
 * merged QKV row.  For each given row (row r of its sample), each part
 * P in {q, k} (q = columns [0, D), k = columns [D, 2D) of the row, where
 * D = n_heads * head_dim; v = columns [2D, 3D) is not read) and each head
 * h (columns [h*head_dim, (h+1)*head_dim) of the part):
 *   ms   = (1/head_dim) * sum_j x[j]^2
 *   n[j] = x[j] / sqrt(ms + eps) * gamma_P[j]          (gamma NULL means 1)
 *   for pair i in [0, head_dim/2):
 *     axis(i) = t if i < sec_t, h if i < sec_t + sec_h, w otherwise
 *     phi     = pos[axis(i)] * theta^(-2i/head_dim)
 *     out[2i]   = n[2i] cos(phi) - n[2i+1] sin(phi)
 *     out[2i+1] = n[2i] sin(phi) + n[2i+1] cos(phi)
 * qkv: the given rows, row k starting at element k * ld_qkv.
 * q_out, k_out: [n_rows, D] doubles.
 */
int oracle_qknorm_rope3d(const void *qkv, int64_t ld_qkv, const void *gamma_q,
                         const void *gamma_k, const int64_t *row_ids,
                         int64_t n_rows, int64_t T, int64_t H, int64_t W,
                         int64_t n_audio, int64_t n_heads, int64_t head_dim,
                         int64_t sec_t, int64_t sec_h, int64_t sec_w,
                         double eps, double theta, int dtype, double *q_out,
                         double *k_out)
{
    int64_t D = n_heads * head_dim;
    int64_t L = T * H * W + n_audio;
    if (n_rows < 0 || T < 0 || H < 0 || W < 0 || n_audio < 0 || L <= 0 ||
        n_heads <= 0 || head_dim <= 0 || head_dim % 2 != 0 || sec_t < 0 ||
        sec_h < 0 || sec_w < 0 || sec_t + sec_h + sec_w != head_dim / 2 ||
        ld_qkv < 2 * D)
        return -1;

    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t g = row_id(row_ids, k);
        int64_t r = g % L;
        int64_t pos[3];
        row_position(r, T, H, W, pos);

        for (int part = 0; part < 2; ++part) {
            const void *gam = part == 0 ? gamma_q : gamma_k;
            double *out = part == 0 ? q_out : k_out;
            for (int64_t hd = 0; hd < n_heads; ++hd) {
                int64_t src = k * ld_qkv + part * D + hd * head_dim;
                int64_t dst = k * D + hd * head_dim;

                double ss = 0.0;
                for (int64_t j = 0; j < head_dim; ++j) {
                    double v = in_val(qkv, src + j, dtype);
                    ss += v * v;
                }
                double denom = sqrt(ss / (double)head_dim + eps);

                for (int64_t i = 0; i < head_dim / 2; ++i) {
                    double a = in_val(qkv, src + 2 * i, dtype) / denom;
                    double b = in_val(qkv, src + 2 * i + 1, dtype) / denom;
                    if (gam) {
                        a = a * in_val(gam, 2 * i, dtype);
                        b = b * in_val(gam, 2 * i + 1, dtype);
                    }
                    int axis = i < sec_t ? 0 : (i < sec_t + sec_h ? 1 : 2);
                    double phi = (double)pos[axis] *
                                 pow(theta, -2.0 * (double)i / (double)head_dim);
                    double c = cos(phi), s = sin(phi);
                    out[dst + 2 * i] = a * c - b * s;
                    out[dst + 2 * i + 1] = a * s + b * c;
                }
            }
        }
    }
    return 0;
}

/*
 * Frequency of rotary pair i.
 *   per_axis = 0: one ladder over all head_dim/2 pairs, theta^(-2i/head_dim),
 *                 the sections only choose the position (M-RoPE style);
 *   per_axis = 1: each section its own ladder over its own 2*s rotary
 *                 dimensions: pair j of a section of s pairs (j counted from
 *                 the section's first pair) has theta^(-2j/(2s)) = theta^(-j/s),
 *                 as when t, h and w each get a RoPE of their own and the
 *                 three are concatenated (an empty section holds no pair, so
 *                 its size is never divided by).
 */
static double rope_freq(int64_t i, int64_t head_dim, int64_t sec_t, int64_t sec_h,
                        double theta, int per_axis)
{
    if (!per_axis)
        return pow(theta, -2.0 * (double)i / (double)head_dim);
    int64_t start, size;
    if (i < sec_t) {
        start = 0;
        size = sec_t;
    } else if (i < sec_t + sec_h) {
        start = sec_t;
        size = sec_h;
    } else {
        start = sec_t + sec_h;
        size = head_dim / 2 - sec_t - sec_h;
    }
    return pow(theta, -(double)(i - start) / (double)size);
}

/*
 * QKNorm + 3D RoPE with a choice of rotary pair layout and of frequency
 * ladder.  half_split = 0 pairs elements (2i, 2i+1) as oracle_qknorm_rope3d
 * does; half_split = 1 pairs element i with element i + head_dim/2 (the
 * "rotate half" layout of GPT-NeoX style implementations):
 *   out[i]              = n[i] cos(phi_i) - n[i + hd/2] sin(phi_i)
 *   out[i + hd/2]       = n[i] sin(phi_i) + n[i + hd/2] cos(phi_i)
 * with phi_i = pos[axis(i)] * rope_freq(i) (per_axis as for rope_freq) and the
 * same sections and positions.  With half_split = 0 and per_axis = 0 this is
 * oracle_qknorm_rope3d itself.  Other arguments as for oracle_qknorm_rope3d.
 */
int oracle_qknorm_rope3d_ex(const void *qkv, int64_t ld_qkv, const void *gamma_q,
                            const void *gamma_k, const int64_t *row_ids, int64_t n_rows,
                            int64_t T, int64_t H, int64_t W, int64_t n_audio,
                            int64_t n_heads, int64_t head_dim, int64_t sec_t,
                            int64_t sec_h, int64_t sec_w, double eps, double theta,
                            int half_split, int per_axis, int dtype, double *q_out,
                            double *k_out)
{
    if (!half_split && !per_axis)
        return oracle_qknorm_rope3d(qkv, ld_qkv, gamma_q, gamma_k, row_ids, n_rows, T, H,
                                    W, n_audio, n_heads, head_dim, sec_t, sec_h, sec_w, eps,
                                    theta, dtype, q_out, k_out);
    int64_t D = n_heads * head_dim;
    int64_t L = T * H * W + n_audio;
    int64_t half = head_dim / 2;
    if (n_rows < 0 || T < 0 || H < 0 || W < 0 || n_audio < 0 || L <= 0 ||
        n_heads <= 0 || head_dim <= 0 || head_dim % 2 != 0 || sec_t < 0 ||
        sec_h < 0 || sec_w < 0 || sec_t + sec_h + sec_w != half || ld_qkv < 2 * D)
        return -1;
    for (int64_t k = 0; k < n_rows; ++k) {
        int64_t r = row_id(row_ids, k) % L;
        int64_t pos[3];
        row_position(r, T, H, W, pos);
        for (int part = 0; part < 2; ++part) {
            const void *gam = part == 0 ? gamma_q : gamma_k;
            double *out = part == 0 ? q_out : k_out;
            for (int64_t hd = 0; hd < n_heads; ++hd) {
                int64_t src = k * ld_qkv + part * D + hd * head_dim;
                int64_t dst = k * D + hd * head_dim;
                double ss = 0.0;
                for (int64_t j = 0; j < head_dim; ++j) {
                    double v = in_val(qkv, src + j, dtype);
                    ss += v * v;
                }
                double denom = sqrt(ss / (double)head_dim + eps);
                for (int64_t i = 0; i < half; ++i) {
                    /* the two elements of pair i */
                    int64_t ia = half_split ? i : 2 * i;
                    int64_t ib = half_split ? i + half : 2 * i + 1;
                    double a = in_val(qkv, src + ia, dtype) / denom;
                    double b = in_val(qkv, src + ib, dtype) / denom;
                    if (gam) {
                        a = a * in_val(gam, ia, dtype);
                        b = b * in_val(gam, ib, dtype);
                    }
                    int axis = i < sec_t ? 0 : (i < sec_t + sec_h ? 1 : 2);
                    double phi = (double)pos[axis] *
                                 rope_freq(i, head_dim, sec_t, sec_h, theta, per_axis);
                    double c = cos(phi), s = sin(phi);
                    out[dst + ia] = a * c - b * s;
                    out[dst + ib] = a * s + b * c;
                }
            }
        }
    }
    return 0;
}

/*
 * Symmetric INT8 quantisation of each head vector (for the INT8 Q/K
 * exchange between GPUs in the KOCPC article's 4x/8x B300 runs):
 *   scale = max_j |x[j]| / 127,  code[j] = round_half_even(x[j] / scale)
 * (scale 0 and all codes 0 for an all-zero head).  x: [n_rows, n_heads *
 * head_dim] doubles; code: same shape (int32 holding values in -127..127);
 * scale: [n_rows, n_heads].
 */
int oracle_quantize_heads(const double *x, int64_t n_rows, int64_t n_heads,
                          int64_t head_dim, int32_t *code, double *scale)
{
    if (n_rows < 0 || n_heads <= 0 || head_dim <= 0)
        return -1;
    for (int64_t k = 0; k < n_rows; ++k) {
        for (int64_t h = 0; h < n_heads; ++h) {
            const double *v = x + (k * n_heads + h) * head_dim;
            int32_t *c = code + (k * n_heads + h) * head_dim;
            double amax = 0.0;
            for (int64_t j = 0; j < head_dim; ++j)
                if (fabs(v[j]) > amax)
                    amax = fabs(v[j]);
            double s = amax / 127.0;
            scale[k * n_heads + h] = s;
            for (int64_t j = 0; j < head_dim; ++j)
                c[j] = s > 0.0 ? (int32_t)nearbyint(v[j] / s) : 0;
        }
    }
    return 0;
}

