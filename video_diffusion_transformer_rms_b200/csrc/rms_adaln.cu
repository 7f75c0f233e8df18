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

// Widen the modulation of (sample, modality) `key` to fp32:
// fac = gamma * (1 + scale), sh = shift, for this thread's slots.
template <typename T, int NT, int VPT>
__device__ __forceinline__ void load_modulation(const RmsArgs &a, int key, int tid,
                                                const bool (&ok)[VPT],
                                                float2 (&fac)[VPT][Io<T>::E / 2],
                                                float2 (&sh)[VPT][Io<T>::E / 2]) {
  using IO = Io<T>;
  constexpr int P = IO::E / 2;
  const int64_t koff = static_cast<int64_t>(key) * a.nvec + tid;
  const uint4 *s0 = static_cast<const uint4 *>(a.scale) + koff;
  const uint4 *h0 = static_cast<const uint4 *>(a.shift) + koff;
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

  int64_t begin;
  int count;  // rows of this CTA's share, walked with local index j
  cta_rows(a.rows, blockIdx.x, gridDim.x, begin, count);
  const int iters = (count + R - 1) / R;
  const unsigned char *xc = xb + begin * row_bytes;
  unsigned char *yc = yb + begin * row_bytes;

  // Copy this thread's slots of iteration `it`'s rows into ring stage s;
  // always commits a group (possibly empty) so the group count is uniform.
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const uint4 *src = reinterpret_cast<const uint4 *>(xc + j * row_bytes) + tid;
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
  int key = -1;                    // 2*b + m those belong to
  int cons = 0;                    // ring stage of iteration `it`
  int buf = 0;                     // which half of `red`
  TokenCursor cur;
  cur.init(begin, a.L);

  for (int it = 0; it < iters; ++it) {
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

    float2 inv2[R];
#pragma unroll
    for (int q = 0; q < R; ++q) inv2[q] = splat2(rsqrtf(fmaf(tot[q], a.inv_D, a.eps)));

    // Fast path: every row of this iteration uses the cached modulation.
    const int nrows = count - it * R < R ? count - it * R : R;
    bool same = true;
    {
      TokenCursor c = cur;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        if (q < nrows) same &= (2 * c.b + (c.r >= a.n_video ? 1 : 0)) == key;
        c.next(a.L);
      }
    }
    if (same) {
#pragma unroll
      for (int q = 0; q < R; ++q) {
        if (q < nrows) {
          uint4 *yrow = reinterpret_cast<uint4 *>(yc + (it * R + q) * row_bytes) + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            if (ok[k]) {
              float2 o[P];
#pragma unroll
              for (int m = 0; m < P; ++m)
                o[m] = fma2(xp[q][k][m], mul2(fac[k][m], inv2[q]), sh[k][m]);
              st_stream16(yrow + k * NT, IO::pack(o));
            }
          }
          cur.next(a.L);
        }
      }
    } else {
      // A modality or sample boundary falls in this iteration: reload the
      // modulation row by row (at most a few times per CTA).
#pragma unroll 1
      for (int q = 0; q < nrows; ++q) {
        const int nkey = 2 * cur.b + (cur.r >= a.n_video ? 1 : 0);
        if (nkey != key) {
          key = nkey;
          load_modulation<T, NT, VPT>(a, key, tid, ok, fac, sh);
        }
        uint4 *yrow = reinterpret_cast<uint4 *>(yc + (it * R + q) * row_bytes) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            float2 o[P];
#pragma unroll
            for (int m = 0; m < P; ++m) {
              // q is not a compile-time index here: select the row's values
              float2 x = xp[0][k][m];
#pragma unroll
              for (int qq = 1; qq < R; ++qq)
                if (q == qq) x = xp[qq][k][m];
              float2 iv = inv2[0];
#pragma unroll
              for (int qq = 1; qq < R; ++qq)
                if (q == qq) iv = inv2[qq];
              o[m] = fma2(x, mul2(fac[k][m], iv), sh[k][m]);
            }
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
