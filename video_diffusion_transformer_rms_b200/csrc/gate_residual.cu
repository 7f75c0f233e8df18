// AdaLN-gated residual add: out = h + gate[b][m] * branch per token row
// (the gate of the adaLN DiT block; one of the elementwise chains the Sol
// Video Inference Engine MiniMax-H3 page removes by fusion).
//
// Same persistent cp.async ring as RMS-AdaLN, with h and branch staged side
// by side and no reduction, so no CTA barrier at all.  The gate vector of
// the current (sample, modality) stays in registers.  HBM traffic:
// read h, read branch, write out = 3*D*esize bytes per row.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

constexpr int kMaxV = 4;

template <typename T, int S>
__global__ void __launch_bounds__(kMaxThreads)
    gate_residual_kernel(const GateArgs a, const int vpt) {
  using IO = Io<T>;
  constexpr int E = IO::E;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4 *ring = reinterpret_cast<uint4 *>(smem);  // [S][2][vpt][threads]

  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;
  const int64_t step = gridDim.x;
  const unsigned char *hb = static_cast<const unsigned char *>(a.h);
  const unsigned char *bb = static_cast<const unsigned char *>(a.branch);
  unsigned char *ob = static_cast<unsigned char *>(a.out);

  auto slot = [&](int s, int which, int k) -> uint4 * {
    return &ring[((s * 2 + which) * vpt + k) * nt + tid];
  };
  auto issue = [&](int64_t r, int s) {
    if (r < a.rows) {
      const uint4 *hs = reinterpret_cast<const uint4 *>(hb + r * row_bytes);
      const uint4 *bs = reinterpret_cast<const uint4 *>(bb + r * row_bytes);
#pragma unroll
      for (int k = 0; k < kMaxV; ++k) {
        const int v = k * nt + tid;
        if (k < vpt && v < a.nvec) {
          cp_async16(slot(s, 0, k), hs + v);
          cp_async16(slot(s, 1, k), bs + v);
        }
      }
    }
    cp_async_commit();
  };

  int64_t row = blockIdx.x;
#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(row + s * step, s);

  uint4 gv[kMaxV];
  int64_t key = -1;
  int cons = 0;
  for (; row < a.rows; row += step) {
    issue(row + (S - 1) * step, cons == 0 ? S - 1 : cons - 1);
    cp_async_wait<S - 1>();

    const int64_t b = row / a.L;
    const int64_t r = row - b * a.L;
    const int64_t nkey = 2 * b + (r >= a.n_video ? 1 : 0);
    if (nkey != key) {
      key = nkey;
      const uint4 *g0 = static_cast<const uint4 *>(a.gate) + key * a.nvec;
#pragma unroll
      for (int k = 0; k < kMaxV; ++k) {
        const int v = k * nt + tid;
        if (k < vpt && v < a.nvec) gv[k] = ld_shared_vec(g0 + v);
      }
    }

    unsigned char *orow = ob + row * row_bytes;
#pragma unroll
    for (int k = 0; k < kMaxV; ++k) {
      const int v = k * nt + tid;
      if (k < vpt && v < a.nvec) {
        float hf[E], bf[E], gf[E], o[E];
        IO::unpack(*slot(cons, 0, k), hf);
        IO::unpack(*slot(cons, 1, k), bf);
        IO::unpack(gv[k], gf);
#pragma unroll
        for (int e = 0; e < E; ++e) o[e] = fmaf(gf[e], bf[e], hf[e]);
        st_stream16(orow + static_cast<int64_t>(v) * 16, IO::pack(o));
      }
    }
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <typename T, int S>
cudaError_t launch_t(const GateArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  const void *fn = reinterpret_cast<const void *>(&gate_residual_kernel<T, S>);
  const size_t smem = static_cast<size_t>(S) * 2 * vpt * threads * 16;
  const int per_sm = resident_blocks(fn, threads, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{threads, vpt, S, smem, static_cast<int>(grid)};
  gate_residual_kernel<T, S><<<static_cast<unsigned>(grid), threads, smem, stream>>>(a, vpt);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_s(const GateArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  const size_t stage = static_cast<size_t>(2) * vpt * threads * 16;
  if (stage <= 24 * 1024) return launch_t<T, 3>(a, threads, vpt, stream, geo);
  return launch_t<T, 2>(a, threads, vpt, stream, geo);
}

}  // namespace

cudaError_t launch_gate_residual(const GateArgs &a, int dtype, cudaStream_t stream,
                                 Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!row_split(a.nvec, kMaxV, kMaxV, kMaxThreads, 32, &threads, &vpt))
    return cudaErrorInvalidValue;
  return dtype == 0 ? launch_s<float>(a, threads, vpt, stream, geo)
                    : launch_s<__nv_bfloat16>(a, threads, vpt, stream, geo);
}

}  // namespace sol
