// Fused RMS-AdaLN (Sol Video Inference Engine MiniMax-H3 page, fusion table,
// row "fused RMS-AdaLN"):
//   y = x / sqrt(mean(x^2) + eps) * gamma * (1 + scale[b][m]) + shift[b][m]
// per token row, m = video/audio modality of the row.
//
// One persistent CTA per resident slot walks rows blockIdx.x, +gridDim.x, ...
// Each row is staged in shared memory by cp.async S-1 rows ahead, reduced in
// fp32 (warp shuffles, then one shared-memory hop across warps) and written
// once.  The modulation vectors of the current (sample, modality) stay in
// registers and are re-read only when a CTA crosses a modality or sample
// boundary, so HBM sees x once and y once: 2*D*esize bytes per row.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

constexpr int kMaxV = 4;  // 16-byte vectors per thread per row

template <typename T, int S, bool GAMMA>
__global__ void __launch_bounds__(kMaxThreads)
    rms_adaln_kernel(const RmsArgs a, const int vpt) {
  using IO = Io<T>;
  constexpr int E = IO::E;
  extern __shared__ __align__(16) unsigned char smem[];
  float *red = reinterpret_cast<float *>(smem);           // [2][32] warp partials
  uint4 *ring = reinterpret_cast<uint4 *>(smem + 256);    // [S][vpt][threads]

  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int nw = nt >> 5;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;
  const int64_t step = gridDim.x;
  const unsigned char *xb = static_cast<const unsigned char *>(a.x);
  unsigned char *yb = static_cast<unsigned char *>(a.y);

  // Copy this thread's slots of row r into ring stage s (always commits a
  // group, possibly empty, so that group counting stays uniform).
  auto issue = [&](int64_t r, int s) {
    if (r < a.rows) {
      const uint4 *src = reinterpret_cast<const uint4 *>(xb + r * row_bytes);
#pragma unroll
      for (int k = 0; k < kMaxV; ++k) {
        const int v = k * nt + tid;
        if (k < vpt && v < a.nvec) cp_async16(&ring[(s * vpt + k) * nt + tid], src + v);
      }
    }
    cp_async_commit();
  };

  int64_t row = blockIdx.x;
#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(row + s * step, s);

  uint4 g[kMaxV];
  if (GAMMA) {
#pragma unroll
    for (int k = 0; k < kMaxV; ++k) {
      const int v = k * nt + tid;
      if (k < vpt && v < a.nvec)
        g[k] = ld_shared_vec(static_cast<const uint4 *>(a.gamma) + v);
    }
  }

  uint4 sc[kMaxV], sh[kMaxV];
  int64_t key = -1;  // 2*b + m of the modulation vectors held in sc / sh
  int cons = 0;      // ring stage holding `row`
  int buf = 0;       // which half of `red`

  for (; row < a.rows; row += step) {
    issue(row + (S - 1) * step, cons == 0 ? S - 1 : cons - 1);
    cp_async_wait<S - 1>();

    const int64_t b = row / a.L;
    const int64_t r = row - b * a.L;
    const int64_t nkey = 2 * b + (r >= a.n_video ? 1 : 0);
    if (nkey != key) {
      key = nkey;
      const uint4 *s0 = static_cast<const uint4 *>(a.scale) + key * a.nvec;
      const uint4 *h0 = static_cast<const uint4 *>(a.shift) + key * a.nvec;
#pragma unroll
      for (int k = 0; k < kMaxV; ++k) {
        const int v = k * nt + tid;
        if (k < vpt && v < a.nvec) {
          sc[k] = ld_shared_vec(s0 + v);
          sh[k] = ld_shared_vec(h0 + v);
        }
      }
    }

    uint4 xv[kMaxV];
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxV; ++k) {
      const int v = k * nt + tid;
      if (k < vpt && v < a.nvec) {
        xv[k] = ring[(cons * vpt + k) * nt + tid];
        float f[E];
        IO::unpack(xv[k], f);
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
      }
    }
    ss = warp_sum(ss);
    if (lane == 0) red[buf * 32 + warp] = ss;
    __syncthreads();
    float tot = 0.f;
    for (int w = 0; w < nw; ++w) tot += red[buf * 32 + w];
    buf ^= 1;
    const float inv = rsqrtf(fmaf(tot, a.inv_D, a.eps));

    unsigned char *yrow = yb + row * row_bytes;
#pragma unroll
    for (int k = 0; k < kMaxV; ++k) {
      const int v = k * nt + tid;
      if (k < vpt && v < a.nvec) {
        float f[E], s[E], t[E], o[E];
        IO::unpack(xv[k], f);
        IO::unpack(sc[k], s);
        IO::unpack(sh[k], t);
        if (GAMMA) {
          float gg[E];
          IO::unpack(g[k], gg);
#pragma unroll
          for (int e = 0; e < E; ++e) o[e] = fmaf(f[e] * inv * gg[e], 1.f + s[e], t[e]);
        } else {
#pragma unroll
          for (int e = 0; e < E; ++e) o[e] = fmaf(f[e] * inv, 1.f + s[e], t[e]);
        }
        st_stream16(yrow + static_cast<int64_t>(v) * 16, IO::pack(o));
      }
    }
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <typename T, int S, bool GAMMA>
cudaError_t launch_t(const RmsArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  const void *fn = reinterpret_cast<const void *>(&rms_adaln_kernel<T, S, GAMMA>);
  const size_t smem = 256 + static_cast<size_t>(S) * vpt * threads * 16;
  const int per_sm = resident_blocks(fn, threads, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{threads, vpt, S, smem, static_cast<int>(grid)};
  rms_adaln_kernel<T, S, GAMMA><<<static_cast<unsigned>(grid), threads, smem, stream>>>(a, vpt);
  return cudaGetLastError();
}

template <typename T, int S>
cudaError_t launch_g(const RmsArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  return a.gamma ? launch_t<T, S, true>(a, threads, vpt, stream, geo)
                 : launch_t<T, S, false>(a, threads, vpt, stream, geo);
}

template <typename T>
cudaError_t launch_s(const RmsArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  // Ring depth by stage size: keep ~3 rows per CTA in flight for rows up to
  // 12 KB, fewer for wider rows so that several CTAs still fit on an SM.
  const size_t stage = static_cast<size_t>(vpt) * threads * 16;
  if (stage <= 12 * 1024) return launch_g<T, 4>(a, threads, vpt, stream, geo);
  return launch_g<T, 2>(a, threads, vpt, stream, geo);
}

}  // namespace

cudaError_t launch_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream, Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!row_split(a.nvec, kMaxV, kMaxV, kMaxThreads, 32, &threads, &vpt))
    return cudaErrorInvalidValue;
  return dtype == 0 ? launch_s<float>(a, threads, vpt, stream, geo)
                    : launch_s<__nv_bfloat16>(a, threads, vpt, stream, geo);
}

}  // namespace sol
