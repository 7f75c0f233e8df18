// Host-side interface between the C ABI (sol_abi.cu) and the kernel
// launchers.  Internal to libsol: arguments arrive here already validated.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace sol {

// Launch geometry of one persistent row-streaming kernel.
struct Geometry {
  int threads;   // CTA size, a multiple of 32
  int vpt;       // 16-byte vectors per thread per row (1 .. max)
  int stages;    // depth of the cp.async ring
  size_t smem;   // dynamic shared memory per CTA
  int grid;      // CTAs (at most one wave of resident CTAs)
};

// CTAs of `kernel` resident per SM at (threads, smem) on the current device;
// raises the kernel's dynamic shared-memory limit once per device.  Returns
// 0 if the configuration cannot be resident (or on a CUDA error, which is
// left for cudaGetLastError).
int resident_blocks(const void *kernel, int threads, size_t smem);

// Streaming multiprocessors of the current device (cached per device).
int device_sms();

// CTA size and 16-byte vectors per thread for a row of `nvec` vectors: the
// smallest CTA of {32, 64, 128, 256} threads that needs at most 6 vectors
// per thread, else 256 threads with up to 8.  Wide per-thread slices keep
// the per-row bookkeeping (one barrier, one reduction, address math) small
// against the streamed bytes.  Returns false if the row does not fit.
bool pick_split(int64_t nvec, int *threads, int *vpt);

// The QKNorm + RoPE kernels prefer more, narrower threads (at most 3
// vectors per thread before growing the CTA, up to 8 at 256 threads): their
// per-vector work is two dependent shuffle reductions long, so they need
// more warps per SM to hide latency than the row-reduction kernels do.  At
// D = 5120 this is 256 threads x 3 vectors (16 warps per SM), which measured
// 3.5% faster than 128 x 5 under sustained load.
bool pick_split_qk(int64_t nvec, int *threads, int *vpt);
#define SOL_QK_SPLITS(X)                                                            \
  X(32, 1) X(32, 2) X(32, 3) X(64, 2) X(64, 3) X(128, 2) X(128, 3) X(256, 2) X(256, 3) \
  X(256, 4) X(256, 5) X(256, 6) X(256, 7) X(256, 8)

// The default (on-the-fly) QKNorm + RoPE kernel: four vectors per thread
// where the row allows, the CTA being the row's vectors / 4 rounded up to a
// whole warp (up to 256 threads), then up to 8 vectors at 256 threads.  At
// D = 5120 that is 160 x 4, which fills every slot.
bool pick_split_otf(int64_t nvec, int *threads, int *vpt);
#define SOL_QK_OTF_SPLITS(X)                                                        \
  X(32, 1) X(32, 2) X(32, 3) X(32, 4) X(64, 4) X(96, 4) X(128, 4) X(160, 4) X(192, 4) \
  X(224, 4) X(256, 4) X(256, 5) X(256, 6) X(256, 7) X(256, 8)

// Table-driven QKNorm + RoPE kernels: two vectors per thread, the CTA being
// the row's vectors / 2 rounded up to the next size below (up to 512
// threads: 320 x 2 at D = 5120), then up to 8 vectors at 256 threads.
bool pick_split_tab(int64_t nvec, int *threads, int *vpt);
#define SOL_QK_TAB_SPLITS(X)                                                           \
  X(32, 1) X(32, 2) X(64, 2) X(96, 2) X(128, 2) X(160, 2) X(192, 2) X(224, 2) X(256, 2) \
  X(320, 2) X(384, 2) X(448, 2) X(512, 2) X(256, 5) X(256, 6) X(256, 7) X(256, 8)

// Interleaved INT8 QKNorm + RoPE (16 elements per lane): `slots` = the
// (head, lane) pairs of one part, n_heads * head_dim / 16.  The smallest CTA
// of {32, 64, 128, 256} threads with at most 5 slots per thread (64 x 5 at
// D = 5120, which measured best: 0.705 ms against 0.77-0.86 ms for 128 x 3,
// 160 x 2 and 320 x 1).
bool pick_split_i8w(int64_t slots, int *threads, int *vpt);
#define SOL_I8W_SPLITS(X)                                                              \
  X(32, 1) X(32, 2) X(32, 3) X(32, 4) X(32, 5) X(64, 3) X(64, 4) X(64, 5) X(128, 3) X(128, 4) \
  X(128, 5) X(256, 3) X(256, 4) X(256, 5)

// Every (threads, vectors per thread) pick_split can return, for the
// launchers' compile-time dispatch.
#define SOL_SPLITS(X)                                                              \
  X(32, 1) X(32, 2) X(32, 3) X(32, 4) X(32, 5) X(32, 6) X(64, 4) X(64, 5) X(64, 6) \
  X(128, 4) X(128, 5) X(128, 6) X(256, 4) X(256, 5) X(256, 6) X(256, 7) X(256, 8)

struct RmsArgs {
  const void *x;       // input rows; with a residual: h
  void *y;
  const void *scale;
  const void *shift;
  const void *gamma;   // may be null
  const void *branch;  // residual only: h_out = h + gate * branch feeds the norm
  const void *gate;    // residual only
  void *h_out;         // residual only
  int64_t rows;       // B * L
  int L;              // < 2^31
  int n_video;
  int nvec;           // 16-byte vectors per row
  float eps;
  float inv_D;
};

struct GateArgs {
  const void *h;
  const void *branch;
  const void *gate;
  void *out;
  int64_t rows;
  int L;
  int n_video;
  int nvec;
};

struct QkArgs {
  const void *qkv;
  void *q_out;
  void *k_out;
  const void *gamma_q;  // may be null
  const void *gamma_k;  // may be null
  int64_t ld_qkv_bytes;
  int64_t ld_out_bytes;
  int64_t rows;       // B * L
  int L;              // < 2^31
  int n_video;        // T * H * W
  int HW;             // H * W
  int H;
  int W;
  int nvec_q;         // 16-byte vectors in q (and in k) of one row
  int npairs;         // head_dim / 2
  int sec_t;          // pairs on the t axis
  int sec_th;         // sec_t + sec_h
  int head_dim;
  float eps;
  float inv_hd;
  float theta;
  // epilogue variants only (sol_qknorm_rope3d_ex): output byte strides per
  // sample, token row and head; per-(row, head) fp32 scales for INT8 output
  int64_t out_sb;
  int64_t out_sr;
  int64_t out_sh;
  float *q_scale;
  float *k_scale;
  int n_heads;
  int per_axis;  // 1: each rotary section its own frequency ladder, theta^(-j/s)
  // table-driven kernels only: rotary table, row p = cos(p*f_i) for every pair
  // i, then sin(p*f_i) (2*npairs floats per row), rows 0 .. n_pos-1
  const float *rope_tab;
};

// Per-head symmetric INT8 quantisation of rows of bf16 head vectors (the v
// columns of merged QKV): codes to out + b*out_sb + r*out_sr + h*out_sh
// (bytes), scales max|x|/127 to scale[(b*L + r)*n_heads + h].
struct QuantArgs {
  const void *src;       // row 0's first element
  int64_t ld_src_bytes;  // row pitch of src
  void *out;
  float *scale;
  int64_t out_sb;
  int64_t out_sr;
  int64_t out_sh;
  int64_t rows;          // B * L
  int L;
  int nvec;              // 16-byte vectors per row (D / 8)
  int n_heads;
};

// First-Block-Cache change detector.  `partial` is the caller's workspace:
// [B][kMaxChangeCtas][2] doubles, every slot a CTA uses rewritten per call.
constexpr int kMaxChangeCtas = 1024;
struct ChangeArgs {
  const void *cur;
  const void *prev;
  void *prev_out;   // may be null (no cache refresh)
  double *out;      // [B + 1][3]: num, den, rel
  double *partial;  // workspace
  int B;
  int L;
  int nvec;
  int ctas_per_sample;  // set by the launcher
};

// GEMM + bias + GELU: C[M, N] = gelu(A[M, K] . B[N, K]^T + bias[N]), bf16.
struct GemmArgs {
  const void *A;
  const void *B;
  const void *bias;  // may be null
  void *C;
  int64_t M, N, K;
};
size_t gemm_gelu_workspace_bytes(const GemmArgs &g);
int gemm_gelu_check(const GemmArgs &g);
cudaError_t launch_gemm_gelu(const GemmArgs &g, void *workspace, cudaStream_t stream);

// dtype: 0 = fp32, 1 = bf16 (sol_dtype).  Each returns the launch error
// (cudaSuccess if the kernel was enqueued) and fills `geo` if non-null.
cudaError_t launch_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream, Geometry *geo);
cudaError_t launch_gate_residual_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream,
                                           Geometry *geo);
cudaError_t launch_gate_residual(const GateArgs &a, int dtype, cudaStream_t stream,
                                 Geometry *geo);
cudaError_t launch_residual_change(const ChangeArgs &a, int dtype, cudaStream_t stream,
                                   Geometry *geo);
// Same, with the partial sums in the library's own device array (no
// workspace): at most kNoAllocMaxSamples samples.
constexpr int kNoAllocMaxSamples = 16;
cudaError_t launch_residual_change_noalloc(ChangeArgs a, int dtype, cudaStream_t stream,
                                           Geometry *geo);
cudaError_t launch_qknorm_rope3d_f32(const QkArgs &a, cudaStream_t stream, Geometry *geo);
cudaError_t launch_qknorm_rope3d_bf16(const QkArgs &a, cudaStream_t stream, Geometry *geo);
// the same reading (cos, sin) from the rotary table a.rope_tab
cudaError_t launch_qknorm_rope3d_tab_f32(const QkArgs &a, cudaStream_t stream, Geometry *geo);
cudaError_t launch_qknorm_rope3d_tab_bf16(const QkArgs &a, cudaStream_t stream, Geometry *geo);
cudaError_t launch_qknorm_rope3d_ex_bf16out(const QkArgs &a, bool half_split, cudaStream_t stream,
                                           Geometry *geo);
cudaError_t launch_qknorm_rope3d_ex_int8out(const QkArgs &a, bool half_split, cudaStream_t stream,
                                           Geometry *geo);
// the same reading (cos, sin) from the rotary table a.rope_tab
cudaError_t launch_qknorm_rope3d_ex_tab_bf16out(const QkArgs &a, bool half_split,
                                               cudaStream_t stream, Geometry *geo);
cudaError_t launch_qknorm_rope3d_ex_tab_int8out(const QkArgs &a, bool half_split,
                                               cudaStream_t stream, Geometry *geo);
// head_dim 64, 128 or 256 (8, 16 or 32 lanes per head).
cudaError_t launch_quantize_heads_int8(const QuantArgs &a, int head_dim, cudaStream_t stream,
                                       Geometry *geo);
inline cudaError_t launch_qknorm_rope3d(const QkArgs &a, int dtype, cudaStream_t stream,
                                        Geometry *geo) {
  if (a.rope_tab)
    return dtype == 0 ? launch_qknorm_rope3d_tab_f32(a, stream, geo)
                      : launch_qknorm_rope3d_tab_bf16(a, stream, geo);
  return dtype == 0 ? launch_qknorm_rope3d_f32(a, stream, geo)
                    : launch_qknorm_rope3d_bf16(a, stream, geo);
}

// Rotary table (row p: cos(p*f_i) for every pair i, then sin(p*f_i)) for the
// table-driven QKNorm + RoPE kernels, computed in fp64, rounded to fp32.
cudaError_t launch_rope_table(float *tab, int n_pos, int npairs, int head_dim, int sec_t,
                              int sec_th, double theta, int per_axis, cudaStream_t stream);

// Limits the launchers accept (checked by the ABI before calling them).
constexpr int64_t kMaxRotaryPairs = 128;     // head_dim <= 256
constexpr int kMaxThreads = 256;
constexpr int64_t kMaxRows = 0x7fffffff;  // B*L, L, H*W: 32-bit row bookkeeping
constexpr int kMaxVpt = 8;
constexpr int64_t kMaxRowBytesRms = 32768;   // D * esize for RMS-AdaLN
constexpr int64_t kMaxRowBytesGate = 32768;  // D * esize for the gated residual
constexpr int64_t kMaxRowBytesQk = 65536;    // 2 * D * esize for QKNorm + RoPE

}  // namespace sol
