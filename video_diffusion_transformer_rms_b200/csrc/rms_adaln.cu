// Fused RMS-AdaLN (Sol Video Inference Engine MiniMax-H3 page, fusion table,
// row "fused RMS-AdaLN"):
//   y = x / sqrt(mean(x^2) + eps) * gamma * (1 + scale[b][m]) + shift[b][m]
// per token row, m = video/audio modality of the row.
//
// One persistent CTA per resident slot walks its own contiguous share of the
// rows, R rows per iteration, so the (sample, modality) of each row follows
// from the previous one without a division.  Thread t owns the 16-byte
// vectors t, t+NT, ... of every row (NT and the vectors per thread are
// compile-time, so all indexing folds to constants).  Rows are staged in
// shared memory by cp.async one iteration ahead; the sums of squares of the
// R rows are reduced together (packed fp32x2 FMAs, warp shuffles, one
// shared-memory hop and one barrier per iteration).
//
// The per-channel factor gamma * (1 + scale) and the shift of the current
// (sample, modality) are widened to fp32 into registers only when the CTA
// crosses a modality or sample boundary; per row each pair of channels then
// costs one packed multiply (factor * inv_rms) and one packed FMA
// (x * that + shift).  HBM sees x once and y once: 2*D*esize bytes per row.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

template <typename T, int NT, int VPT, int R, int S>
__global__ void __launch_bounds__(NT) rms_adaln_kernel(const RmsArgs a) {
  using IO = Io<T>;
  constexpr int P = IO::E / 2;  // fp32 pairs per 16-byte vector
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  float *red = reinterpret_cast<float *>(smem);                       // [2][R][32]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + 2 * R * 32 * 4);    // [S][R][VPT][NT]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;
  const unsigned char *xb = static_cast<const unsigned char *>(a.x);
  unsigned char *yb = static_cast<unsigned char *>(a.y);

  bool ok[VPT];  // slot k holds vector k*NT + tid of the row
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = k * NT + tid < a.nvec;

  for (int i = tid; i < 2 * R * 32; i += NT) red[i] = 0.f;  // unused warp slots read 0
  __syncthreads();

  int64_t begin, end;
  cta_rows(a.rows, blockIdx.x, gridDim.x, begin, end);
  const int64_t iters = (end - begin + R - 1) / R;

  // Copy this thread's slots of iteration `it`'s rows into ring stage s;
  // always commits a group (possibly empty) so the group count is uniform.
  auto issue = [&](int64_t it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int64_t row = begin + it * R + q;
      if (it < iters && row < end) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xb + row * row_bytes) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k)
          if (ok[k]) cp_async16(&ring[((s * R + q) * VPT + k) * NT + tid], src + k * NT);
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);

  float2 fac[VPT][P], sh[VPT][P];  // gamma*(1+scale) and shift of `key`
  int64_t key = -1;                // 2*b + m those belong to
  int cons = 0;                    // ring stage of iteration `it`
  int buf = 0;                     // which half of `red`
  TokenCursor cur;
  cur.init(begin, a.L);

  for (int64_t it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);
    cp_async_wait<S - 1>();

    float2 xp[R][VPT][P];
    float tot[R];
#pragma unroll
    for (int q = 0; q < R; ++q) {
      float2 acc = splat2(0.f);
#pragma unroll
      for (int k = 0; k < VPT; ++k) {
        if (ok[k]) {
          IO::unpack(ring[((cons * R + q) * VPT + k) * NT + tid], xp[q][k]);
#pragma unroll
          for (int m = 0; m < P; ++m) acc = fma2(xp[q][k][m], xp[q][k][m], acc);
        }
      }
      tot[q] = warp_sum(acc.x + acc.y);
    }
    if (NW > 1) {
      if (lane == 0) {
#pragma unroll
        for (int q = 0; q < R; ++q) red[(buf * R + q) * 32 + warp] = tot[q];
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < R; ++q) {
        const float4 *r4 = reinterpret_cast<const float4 *>(red + (buf * R + q) * 32);
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < (NW + 3) / 4; ++w) {
          const float4 v = r4[w];
          t += (v.x + v.y) + (v.z + v.w);
        }
        tot[q] = t;
      }
      buf ^= 1;
    }

#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int64_t row = begin + it * R + q;
      if (row < end) {
        const int64_t nkey = 2 * cur.b + (cur.r >= a.n_video ? 1 : 0);
        if (nkey != key) {
          key = nkey;
          const uint4 *s0 = static_cast<const uint4 *>(a.scale) + key * a.nvec + tid;
          const uint4 *h0 = static_cast<const uint4 *>(a.shift) + key * a.nvec + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            if (ok[k]) {
              float2 sc[P];
              IO::unpack(ld_shared_vec(s0 + k * NT), sc);
              IO::unpack(ld_shared_vec(h0 + k * NT), sh[k]);
#pragma unroll
              for (int m = 0; m < P; ++m) fac[k][m] = add2(sc[m], splat2(1.f));
              if (a.gamma) {
                float2 g[P];
                IO::unpack(ld_shared_vec(static_cast<const uint4 *>(a.gamma) + k * NT + tid), g);
#pragma unroll
                for (int m = 0; m < P; ++m) fac[k][m] = mul2(fac[k][m], g[m]);
              }
            }
          }
        }
        const float2 inv2 = splat2(rsqrtf(fmaf(tot[q], a.inv_D, a.eps)));
        uint4 *yrow = reinterpret_cast<uint4 *>(yb + row * row_bytes) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            float2 o[P];
#pragma unroll
            for (int m = 0; m < P; ++m) o[m] = fma2(xp[q][k][m], mul2(fac[k][m], inv2), sh[k][m]);
            st_stream16(yrow + k * NT, IO::pack(o));
          }
        }
        cur.next(a.L);
      }
    }
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <typename T, int NT, int VPT>
cudaError_t launch_t(const RmsArgs &a, cudaStream_t stream, Geometry *geo) {
  constexpr int R = VPT <= 6 ? 2 : 1;  // two rows per iteration while registers allow
  constexpr int S = 2;
  const void *fn = reinterpret_cast<const void *>(&rms_adaln_kernel<T, NT, VPT, R, S>);
  const size_t smem = 2 * R * 32 * 4 + static_cast<size_t>(S) * R * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  rms_adaln_kernel<T, NT, VPT, R, S><<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(const RmsArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch_t<T, NT, V>(a, stream, geo);
  SOL_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream, Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!pick_split(a.nvec, &threads, &vpt)) return cudaErrorInvalidValue;
  return dtype == 0 ? dispatch<float>(a, threads, vpt, stream, geo)
                    : dispatch<__nv_bfloat16>(a, threads, vpt, stream, geo);
}

}  // namespace sol
