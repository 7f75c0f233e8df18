// Rotary table for the table-driven QKNorm + 3D RoPE kernels (rotary
// embedding of RoFormer, frequency list split into t / h / w sections as in
// the multimodal RoPE of the MiniMax-H3 page's "fused QKNorm + RoPE" row).
//
// Positions are integers on every axis, so the (cos, sin) of every rotary
// angle a call can meet is a function of (position, pair) alone: row p of
// the table holds cos(p * f_i) for the npairs pairs i, then sin(p * f_i).
// f_i is theta^(-2i/head_dim) (one ladder over all pairs), or with the
// per-axis flag theta^(-j/s) for local pair j of a section of s pairs.  The
// angle and its sine and cosine are computed in fp64 (CUDA's sincos reduces
// the argument exactly) and rounded once to fp32, so an entry is within half
// an fp32 ulp of the exact value.  Built once per (n_pos, head_dim,
// sections, theta, flag) and reused by every layer and denoising step.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

__global__ void rope_table_kernel(float *tab, int n_pos, int npairs, int head_dim, int sec_t,
                                  int sec_th, double theta, int per_axis) {
  const int64_t n = static_cast<int64_t>(n_pos) * npairs;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(i / npairs);  // position
    const int j = static_cast<int>(i - static_cast<int64_t>(p) * npairs);  // pair
    double e = -2.0 * j / head_dim;
    if (per_axis) {
      const int start = j < sec_t ? 0 : (j < sec_th ? sec_t : sec_th);
      const int size = j < sec_t ? sec_t : (j < sec_th ? sec_th - sec_t : npairs - sec_th);
      e = -static_cast<double>(j - start) / size;
    }
    double s, c;
    sincos(static_cast<double>(p) * pow(theta, e), &s, &c);
    float *row = tab + static_cast<int64_t>(p) * 2 * npairs;
    row[j] = static_cast<float>(c);
    row[npairs + j] = static_cast<float>(s);
  }
}

}  // namespace

cudaError_t launch_rope_table(float *tab, int n_pos, int npairs, int head_dim, int sec_t,
                              int sec_th, double theta, int per_axis, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(n_pos) * npairs;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (n + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(device_sms()) * 8;
  if (cap > 0 && blocks > cap) blocks = cap;
  rope_table_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      tab, n_pos, npairs, head_dim, sec_t, sec_th, theta, per_axis);
  return cudaGetLastError();
}

}  // namespace sol
