/*
 * sol.h - C ABI of libsol, the fused per-token hot path of a joint
 * video+audio diffusion-transformer block on NVIDIA B200 (sm_100a).
 *
 * The three operations of the per-token path, each one kernel launch (the
 * variants and next steps are declared further down):
 *   sol_rms_adaln      RMSNorm then AdaLN modulation  x^ * (1 + scale) + shift
 *   sol_gate_residual  AdaLN-gated residual add        h + gate * branch
 *   sol_qknorm_rope3d  per-head RMS norm of q and k, then 3D multimodal RoPE
 *
 * The fusions are the ones the Sol Video Inference Engine MiniMax-H3
 * on-device page lists in its fusion table ("fused RMS-AdaLN": no HBM
 * round-trips across the modulation branch; "fused QKNorm + RoPE": no
 * separate read/write passes over Q and K, no separate 3D MM-RoPE indexing);
 * the KOCPC Sol-H3 article repeats them in "Technical Composition".  The
 * gated residual is one of the elementwise steps that the same page leaves to
 * its torch.compile row: the adaLN gate of the DiT block.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Token rows.  A batch holds B samples of L rows each, row-major and
 * contiguous: row r of sample b is global row b*L + r.  In every sample the
 * first n_video rows are video latent patches (raster order, t-major, for
 * sol_qknorm_rope3d n_video = T*H*W) and the remaining L - n_video rows are
 * audio tokens (the joint single-stream sequence of the H3-Omni transformer).
 * Row r is "video" (modality 0) if r < n_video, else "audio" (modality 1).
 *
 * Modulation vectors.  scale, shift and gate are [B, 2, D] arrays: index
 * [b][0] holds sample b's video vector and [b][1] its audio vector.
 *
 * Element type.  All tensor arguments of one call have the same type:
 * SOL_BF16 (bfloat16) or SOL_F32.  Arithmetic is fp32 inside the kernels;
 * outputs are rounded once, to nearest even.
 *
 * Memory.  Every tensor pointer is a DEVICE pointer (cudaMalloc'd, managed,
 * or mapped so the GPU can read it) on the current device, 16-byte aligned,
 * with every row start 16-byte aligned (so D, and the row strides, must be
 * multiples of 8 elements for bf16 and 4 for fp32).  The caller owns all
 * buffers.  The library allocates nothing, keeps no per-call state and may be
 * called from several host threads at once.
 *
 * Aliasing.  An output may be exactly its input (in place) as stated per
 * call; any other overlap between an output and another argument is rejected
 * with SOL_ERR_INVALID_ARG.
 *
 * Streams and errors.  Each call validates its arguments on the host, then
 * enqueues one kernel on `stream` (NULL = the legacy default stream) and
 * returns without synchronising.  On any non-OK status nothing has been
 * enqueued, except SOL_ERR_CUDA, which reports a failed launch (the CUDA
 * error was read and cleared with cudaGetLastError).  A call with zero rows
 * is a no-op that returns SOL_OK.  sol_last_error() gives a one-line reason
 * for the calling thread's last non-OK status.
 */
#ifndef SOL_H
#define SOL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */
typedef struct CUstream_st *sol_stream_t;

typedef enum sol_status {
    SOL_OK = 0,
    SOL_ERR_INVALID_ARG = 1, /* null pointer, bad size, or forbidden overlap */
    SOL_ERR_MISALIGNED = 2,  /* a pointer or row start not 16-byte aligned */
    SOL_ERR_UNSUPPORTED = 3, /* valid but outside the built kernels' limits */
    SOL_ERR_CUDA = 4         /* the CUDA runtime reported an error */
} sol_status;

typedef enum sol_dtype {
    SOL_F32 = 0,
    SOL_BF16 = 1
} sol_dtype;

/*
 * Fused RMS-AdaLN (fusion table of the Sol Video Inference Engine MiniMax-H3
 * page, row "fused RMS-AdaLN"; RMSNorm of Zhang & Sennrich, adaLN modulation
 * of the DiT block).  For every row of sample b with modality m:
 *
 *   y[c] = x[c] / sqrt(mean_c(x^2) + eps) * gamma[c] * (1 + scale[b][m][c])
 *          + shift[b][m][c]
 *
 *   x, y          [B, L, D] device, contiguous.  y may equal x (in place).
 *   scale, shift  [B, 2, D] device.
 *   gamma         [D] device, or NULL for a weight of 1 (the adaLN norm of a
 *                 DiT block has no learnable weight; the option is kept).
 *   n_video       0 <= n_video <= L.
 *   D             > 0; at most 16384 (bf16) / 8192 (fp32)
 *                 (SOL_ERR_UNSUPPORTED beyond).
 *   eps           >= 0, added inside the square root (1e-6 in the model).
 */
sol_status sol_rms_adaln(const void *x, void *y, const void *scale,
                         const void *shift, const void *gamma, int64_t B,
                         int64_t L, int64_t n_video, int64_t D, float eps,
                         sol_dtype dtype, sol_stream_t stream);

/*
 * AdaLN-gated residual add (the adaLN gate of the DiT block; one of the
 * elementwise steps the Sol pages leave to torch.compile capture).  For every
 * row of sample b with modality m:
 *
 *   out[c] = h[c] + gate[b][m][c] * branch[c]
 *
 *   h, branch, out [B, L, D] device, contiguous.  out may equal h or branch.
 *   gate           [B, 2, D] device.
 *   n_video, D     as for sol_rms_adaln (same D limit).
 */
sol_status sol_gate_residual(const void *h, const void *branch,
                             const void *gate, void *out, int64_t B, int64_t L,
                             int64_t n_video, int64_t D, sol_dtype dtype,
                             sol_stream_t stream);

/*
 * Fused AdaLN-gated residual + RMS-AdaLN: the block's "h = h + gate * attn;
 * x = RMS-AdaLN(h)" chain in one pass (an elementwise step of the pages'
 * torch.compile row fused into the fused RMS-AdaLN row of the Sol Video
 * Inference Engine MiniMax-H3 fusion table).  For every row of
 * sample b with modality m:
 *
 *   h_out[c] = h[c] + gate[b][m][c] * branch[c]
 *   y[c]     = h_out[c] / sqrt(mean_c(h_out^2) + eps) * gamma[c]
 *              * (1 + scale[b][m][c]) + shift[b][m][c]
 *
 * The normalisation reads h_out before it is rounded to the I/O type.  HBM
 * traffic per row is 4*D elements instead of 5*D for sol_gate_residual
 * followed by sol_rms_adaln.
 *
 *   h, branch, h_out, y  [B, L, D] device, contiguous.  h_out may equal h
 *                        (in place); y must not overlap any other argument.
 *   gate, scale, shift   [B, 2, D] device.
 *   gamma, n_video, D, eps  as for sol_rms_adaln (same D limit).
 */
sol_status sol_gate_residual_rms_adaln(const void *h, const void *branch,
                                       const void *gate, void *h_out, void *y,
                                       const void *scale, const void *shift,
                                       const void *gamma, int64_t B, int64_t L,
                                       int64_t n_video, int64_t D, float eps,
                                       sol_dtype dtype, sol_stream_t stream);

/*
 * Fused per-head QKNorm + 3D multimodal RoPE on a merged QKV projection
 * (fusion table of the Sol Video Inference Engine MiniMax-H3 page, rows
 * "fused QKNorm + RoPE" and "QKV merge"; RoPE of Su et al., RoFormer).
 *
 * Each row holds q in columns [0, D), k in [D, 2D) (v, if present after
 * them, is neither read nor written), D = n_heads * head_dim; head j of q or
 * k is columns [j*head_dim, (j+1)*head_dim) of that part.  For each head:
 *
 *   n[c]  = x[c] / sqrt(mean_c(x^2) + eps) * gamma_P[c]   (P = q or k)
 *   pair i = (n[2i], n[2i+1]), i < head_dim/2, rotated by
 *   phi_i = pos_a(i) * theta^(-2i/head_dim):
 *     out[2i]   = n[2i] cos(phi_i) - n[2i+1] sin(phi_i)
 *     out[2i+1] = n[2i] sin(phi_i) + n[2i+1] cos(phi_i)
 *   with a(i) = t for i < sec_t, h for i < sec_t + sec_h, else w.
 *
 * Positions (per sample, the same for every sample): video row r < T*H*W
 * has (t, h, w) = (r / (H*W), (r / W) mod H, r mod W); audio row
 * i = r - T*H*W has (i, 0, 0).  So L = T*H*W + n_audio.
 *
 *   qkv          device; row g (= b*L + r) starts at qkv + g*ld_qkv elements;
 *                ld_qkv >= 2*D (3*D for a packed [.., 3D] projection).
 *   q_out, k_out device; row g of q (k) goes to q_out (k_out) + g*ld_out.
 *                ld_out >= D.  In place: q_out == qkv, k_out == qkv + D and
 *                ld_out == ld_qkv.  Otherwise q_out and k_out must not
 *                overlap qkv's rows nor each other (q_out = buf,
 *                k_out = buf + D, ld_out = 2*D is fine).
 *   gamma_q, gamma_k [head_dim] device, or NULL for a weight of 1; one
 *                vector for all heads.
 *   head_dim     even, head_dim / (8 for bf16, 4 for fp32) a power of two
 *                in [2, 32] (so 16..256 bf16, 8..128 fp32), else
 *                SOL_ERR_UNSUPPORTED; sec_t + sec_h + sec_w == head_dim / 2.
 *   n_heads      > 0, with D at most 16384 (bf16) / 8192 (fp32)
 *                (SOL_ERR_UNSUPPORTED beyond).
 *   eps >= 0; theta > 0 (10000 in the model).
 *   T, H, W, n_audio >= 0, B >= 0.
 */
sol_status sol_qknorm_rope3d(const void *qkv, int64_t ld_qkv, void *q_out,
                             void *k_out, int64_t ld_out, const void *gamma_q,
                             const void *gamma_k, int64_t B, int64_t T,
                             int64_t H, int64_t W, int64_t n_audio,
                             int64_t n_heads, int64_t head_dim, int64_t sec_t,
                             int64_t sec_h, int64_t sec_w, float eps,
                             float theta, sol_dtype dtype,
                             sol_stream_t stream);

/*
 * Output layout and epilogue of sol_qknorm_rope3d_ex.
 *
 * Element (sample b, token row r, head h, channel c) of q (k) goes to
 * q_out (k_out) + b*stride_b + r*stride_row + h*stride_head + c, strides in
 * elements of the output type, channels contiguous.  [B, L, H, hd] is
 * (L*H*hd, H*hd, hd); attention's [B, H, L, hd] is (H*L*hd, hd, L*hd).
 * The strides must address distinct elements (not checked).
 */
typedef struct sol_qk_layout {
    int64_t stride_b;
    int64_t stride_row;
    int64_t stride_head;
    int32_t half_split; /* 0: pair i = (2i, 2i+1); 1: pair i = (i, i + hd/2) */
    int32_t int8_out;   /* 1: q_out/k_out receive int8 codes, and q_scale /
                           k_scale [B, L, H] fp32 receive max|x| / 127 per head */
    float *q_scale;     /* int8_out only: device, 4-byte aligned */
    float *k_scale;
    int32_t per_axis_freq; /* 0: one frequency ladder over all head_dim/2
                              pairs, theta^(-2i/head_dim), the sections only
                              choosing the position; 1: each section a ladder
                              of its own, local pair j of a section of s pairs
                              at theta^(-j/s) (t, h and w each a RoPE over
                              their own 2s dimensions) */
    int32_t reserved;   /* must be 0 */
    void *v_out;        /* int8_out only, may be NULL: if set, v (columns
                           [2D, 3D) of qkv) is quantised as it stands (no
                           norm, no rotation) to int8 codes here, in the
                           layout of q_out/k_out, with scales in v_scale */
    float *v_scale;     /* [B, L, H] fp32, with v_out */
} sol_qk_layout;

/*
 * QKNorm + 3D RoPE (as sol_qknorm_rope3d) with the epilogue variants its
 * consumers need: any head-strided output layout (attention's [B, H, L, hd]
 * directly), the half-split rotary pair layout, and INT8 output with
 * symmetric per-(row, head) scales, code = round_half_even(x * 127 /
 * max|x|) in fp32 (the quantised Q/K the KOCPC Sol-H3 article's 4x/8x B300
 * runs exchange between GPUs).  The rotation angles, sections, positions,
 * gamma and eps are those of sol_qknorm_rope3d.
 *
 *   dtype       SOL_BF16 input (SOL_ERR_UNSUPPORTED otherwise); output bf16,
 *               or int8 with int8_out.
 *   head_dim    64, 128 or 256.
 *   q_out, k_out, layout   see sol_qk_layout; outputs must not overlap qkv,
 *               each other or the scales (no in-place form).  Each output
 *               vector start (16 bytes, 8 for int8) must be aligned to its
 *               size: base and strides * element size multiples of it.
 *               v_out / v_scale follow the int8 rules of q_out / q_scale and
 *               must overlap none of the other buffers; with v_out set,
 *               ld_qkv must be >= 3*D.  The quantisation of v is a second
 *               kernel on the same stream (v is not read by the first).
 *   other arguments as for sol_qknorm_rope3d.
 *
 * The per-axis frequency ladder and the quantised v are options of this
 * library (the pages name per-axis frequencies and INT8 Q/K/V transfer, not
 * their exact form).  A layout with reserved != 0 or per_axis_freq outside
 * {0, 1} returns SOL_ERR_INVALID_ARG; v_out without int8_out returns
 * SOL_ERR_UNSUPPORTED.
 */
sol_status sol_qknorm_rope3d_ex(const void *qkv, int64_t ld_qkv, void *q_out,
                                void *k_out, const sol_qk_layout *layout,
                                const void *gamma_q, const void *gamma_k,
                                int64_t B, int64_t T, int64_t H, int64_t W,
                                int64_t n_audio, int64_t n_heads,
                                int64_t head_dim, int64_t sec_t, int64_t sec_h,
                                int64_t sec_w, float eps, float theta,
                                sol_dtype dtype, sol_stream_t stream);

/*
 * Precomputed rotary table for the table-driven QKNorm + 3D RoPE entry
 * points (the "3D MM-RoPE indexing" of the MiniMax-H3 page's "fused QKNorm +
 * RoPE" row, done once instead of per row).
 *
 * Rotary positions are integers on every axis (t, h, w, and the audio index
 * on t), so every (cos, sin) a call needs is a function of (position p,
 * pair i) alone.  Row p of the table holds cos(p * f_i) for the head_dim/2
 * pairs i, then sin(p * f_i): head_dim floats per row, n_pos rows.  f_i is
 * theta^(-2i/head_dim), or with per_axis_freq theta^(-j/s) for local pair j
 * of a section of s pairs (as sol_qk_layout.per_axis_freq).  Angles, sines
 * and cosines are computed in fp64 and rounded once to fp32.
 *
 * The table depends only on these fields: build it once per video shape and
 * reuse it for every layer and denoising step.  The caller owns `data`.
 */
typedef struct sol_rope_table {
    float *data;        /* device, sol_rope_table_bytes(n_pos, head_dim)
                           bytes, 16-byte aligned */
    int64_t n_pos;      /* rows: positions 0 .. n_pos - 1 on every axis */
    int64_t head_dim;   /* even, 2 .. 256 */
    int64_t sec_t;      /* rotary pairs on t, h and w; sum = head_dim / 2 */
    int64_t sec_h;
    int64_t sec_w;
    float theta;        /* > 0 */
    int32_t per_axis_freq; /* 0 or 1, as in sol_qk_layout */
} sol_rope_table;

/* Bytes of a rotary table: n_pos * head_dim * 4 (0 if n_pos < 0, head_dim
 * is odd or not in [2, 256], or the size overflows). */
size_t sol_rope_table_bytes(int64_t n_pos, int64_t head_dim);

/*
 * Fill tab->data on `stream` (one kernel).  SOL_ERR_INVALID_ARG for a null
 * table or data, n_pos < 0 or beyond 2^31 - 1, a bad head_dim, sections
 * that do not sum to head_dim / 2, theta <= 0 or per_axis_freq outside
 * {0, 1}; SOL_ERR_MISALIGNED if data is not 16-byte aligned.  n_pos = 0 is
 * a no-op.
 */
sol_status sol_rope_table_build(const sol_rope_table *tab, sol_stream_t stream);

/*
 * sol_qknorm_rope3d with the rotation's (cos, sin) read from a rotary table
 * built by sol_rope_table_build (on the same stream, or ordered before this
 * call) instead of being computed per row.  head_dim, the sections, theta
 * and the frequency rule are the table's; the other arguments and rules are
 * those of sol_qknorm_rope3d.  The kernel does no per-row angle work (no
 * fp64 reduction, no sine or cosine): at the 5 s clip shape it ran 0.80 ms
 * against 0.82 ms for sol_qknorm_rope3d on a B200.
 *
 *   tab   host pointer to the descriptor; tab->data is read by the kernel.
 *         Every position the call meets must be a table row:
 *         n_pos >= max(T, H, W) when T*H*W > 0, and n_pos >= n_audio
 *         (SOL_ERR_INVALID_ARG otherwise).  The outputs must not overlap
 *         the table.
 * Results differ from sol_qknorm_rope3d's by the rounding of the table
 * (fp64-exact (cos, sin) rounded once to fp32, against sincosf of the
 * fp64-reduced angle), i.e. within an fp32 ulp or two before the bf16
 * rounding of the output.
 */
sol_status sol_qknorm_rope3d_tab(const void *qkv, int64_t ld_qkv, void *q_out,
                                 void *k_out, int64_t ld_out,
                                 const void *gamma_q, const void *gamma_k,
                                 const sol_rope_table *tab, int64_t B,
                                 int64_t T, int64_t H, int64_t W,
                                 int64_t n_audio, int64_t n_heads, float eps,
                                 sol_dtype dtype, sol_stream_t stream);

/*
 * sol_qknorm_rope3d_ex with the rotation read from a rotary table, as
 * sol_qknorm_rope3d_tab.  layout->per_axis_freq must equal
 * tab->per_axis_freq (SOL_ERR_INVALID_ARG otherwise); head_dim, sections
 * and theta are the table's; everything else as sol_qknorm_rope3d_ex.
 */
sol_status sol_qknorm_rope3d_ex_tab(const void *qkv, int64_t ld_qkv,
                                    void *q_out, void *k_out,
                                    const sol_qk_layout *layout,
                                    const void *gamma_q, const void *gamma_k,
                                    const sol_rope_table *tab, int64_t B,
                                    int64_t T, int64_t H, int64_t W,
                                    int64_t n_audio, int64_t n_heads,
                                    float eps, sol_dtype dtype,
                                    sol_stream_t stream);

/*
 * First-Block-Cache change detector (Sol Video Inference Engine MiniMax-H3
 * page, cross-step caching paragraph: the first block's residual is compared
 * with the previous denoising step's, and the remaining blocks are skipped
 * when it has barely moved, against one residual-difference threshold).
 * Relative L1 difference per sample b and over the whole batch:
 *
 *   num_b = sum_{r,c} |cur[b][r][c] - prev[b][r][c]|
 *   den_b = sum_{r,c} |prev[b][r][c]|
 *   rel_b = num_b / den_b   (0 if num_b = den_b = 0; +inf if only den_b = 0)
 *
 * and, if prev_out is non-null, prev_out = cur in the same pass (the cache
 * refresh a step that does not skip performs).
 *
 *   cur, prev    [B, L, D] device, contiguous, 16-byte aligned.
 *   prev_out     [B, L, D] device or NULL; may equal prev (in place), else
 *                must not overlap cur or prev.
 *   out          device, (B + 1) * 3 doubles, 8-byte aligned: row b is
 *                (num_b, den_b, rel_b), row B the batch (sum of num, sum of
 *                den, their ratio).  Sums are accumulated in fp32 per row
 *                (at most 64 terms) and fp64 beyond, in a fixed order: the
 *                result is deterministic.
 *   workspace    device scratch of at least
 *                sol_residual_change_workspace_bytes(B) bytes, 16-byte
 *                aligned, owned by the caller; its contents on entry do not
 *                matter and are overwritten.  Calls that share a workspace
 *                must be ordered on one stream.
 *   D            as for sol_rms_adaln (same limit); B <= 65535, B*L < 2^31.
 * Two kernels are enqueued (partial sums, then a one-CTA finalisation).
 */
sol_status sol_residual_change(const void *cur, const void *prev,
                               void *prev_out, int64_t B, int64_t L, int64_t D,
                               double *out, void *workspace,
                               size_t workspace_bytes, sol_dtype dtype,
                               sol_stream_t stream);

/* Workspace bytes sol_residual_change needs for B samples (a pure function
 * of B; 16 KiB per sample). */
size_t sol_residual_change_workspace_bytes(int64_t B);

/*
 * sol_residual_change without a workspace argument.  This entry point has no
 * counterpart on the pages; it exists for callers that cannot call
 * cudaMalloc: a host that has already handed the device's memory to its own
 * pool or framework allocator (so a raw cudaMalloc would fail or fragment
 * it), a hot loop that must not pay cudaMalloc/cudaFree's implicit device
 * synchronisation, or a plain-C plug-in with no allocator to borrow from.
 *
 * It computes exactly what sol_residual_change computes (same kernels, same
 * fixed summation order) and allocates nothing.  The partial sums live in
 * one device array inside libsol, 256 KiB, enough for B <= 16 samples; every
 * GPU that loads the library holds that array until the process exits.
 * Larger B returns SOL_ERR_UNSUPPORTED (use sol_residual_change).
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture.  The address is kept for the life of the
 * process: a cudaDeviceReset of that device makes it stale (the library may
 * be loaded again elsewhere in device memory), so do not call this entry
 * point on a device after resetting it; use sol_residual_change there.  Every call shares the one array and it keeps
 * the last call's contents; each call rewrites every slot it later reads,
 * so nothing needs clearing, but calls whose kernels overlap on the GPU
 * (different streams, or different host threads on one device) race on it:
 * order them on one stream.
 *
 *   cur, prev, prev_out, B, L, D, out, dtype: as for sol_residual_change.
 */
sol_status sol_residual_change_noalloc(const void *cur, const void *prev,
                                       void *prev_out, int64_t B, int64_t L,
                                       int64_t D, double *out, sol_dtype dtype,
                                       sol_stream_t stream);

/*
 * GEMM + bias + GELU in one kernel (Sol Video Inference Engine MiniMax-H3
 * page, fusion table, row "GEMM + GELU": the MLP's activation-sized HBM round
 * trip removed by applying GELU in the GEMM epilogue):
 *
 *   C[m][n] = gelu(sum_k A[m][k] * B[n][k] + bias[n]),
 *   gelu(x) = 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))
 *
 * on the 5th-generation tensor cores (tcgen05 MMA, fp32 accumulators in
 * tensor memory, TMA-staged operands).
 *
 *   A        [M, K] bf16 device, row-major (tokens).
 *   B        [N, K] bf16 device, row-major (a Linear layer's weight).
 *   bias     [N] bf16 device, or NULL.
 *   C        [M, N] bf16 device, row-major; must not overlap A, B or bias.
 *   M >= 0 (0 is a no-op), N, K > 0, each below 2^31; N and K multiples of
 *   8 (16-byte rows); pointers 16-byte aligned.
 *   workspace, workspace_bytes  device scratch of at least
 *            sol_gemm_gelu_workspace_bytes(M, N, K) bytes (may be NULL/0 when
 *            that is 0), owned by the caller.
 */
sol_status sol_gemm_gelu(const void *A, const void *B, const void *bias,
                         void *C, int64_t M, int64_t N, int64_t K,
                         void *workspace, size_t workspace_bytes,
                         sol_stream_t stream);

/* Workspace bytes sol_gemm_gelu needs for this problem on the current device. */
size_t sol_gemm_gelu_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Static, human-readable name of a status code. */
const char *sol_status_string(sol_status status);

/* One-line reason for the calling thread's most recent non-OK status, or ""
 * if its last call succeeded.  The pointer stays valid until the thread's
 * next libsol call. */
const char *sol_last_error(void);

/* ABI version, (major << 16) | minor.  2.0: sol_qk_layout gained
 * per_axis_freq, reserved, v_out and v_scale (a larger struct; callers built
 * against 1.x must be rebuilt).  2.1: the rotary table (sol_rope_table,
 * sol_qknorm_rope3d_tab, sol_qknorm_rope3d_ex_tab). */
int sol_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SOL_H */
