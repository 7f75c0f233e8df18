// Fused RMS-AdaLN (Sol Video Inference Engine MiniMax-H3 page, fusion table,
// row "fused RMS-AdaLN"):
//   y = x / sqrt(mean(x^2) + eps) * gamma * (1 + scale[b][m]) + shift[b][m]
// per token row, m = video/audio modality of the row; and the same with the
// AdaLN-gated residual in front of it (the block's "h = h + gate * attn;
// x = RMS-AdaLN(h)" chain), where x = h + gate[b][m] * branch is formed in
// registers, written once as h_out and normalised without a round trip
// through HBM.
//
// One persistent CTA per resident slot walks its rows (chunks of kRmsChunk
// consecutive rows dealt round-robin over the CTAs), R rows per iteration,
// so the (sample, modality) of each row follows from the previous one
// without a division inside a chunk.  Thread t owns the 16-byte
// vectors t, t+NT, ... of every row (NT and the vectors per thread are
// compile-time, so all indexing folds to constants).  Rows are staged in
// shared memory by cp.async one iteration ahead; the sums of squares of the
// R rows are reduced together (packed fp32x2 FMAs, warp shuffles, one
// shared-memory hop and one barrier per iteration).
//
// The per-channel factor gamma * (1 + scale), the shift and (with the
// residual) the gate of the current (sample, modality) are widened to fp32
// into registers only when the CTA crosses a modality or sample boundary.
// Iterations whose rows all share the cached modulation take a fast path;
// an iteration that straddles a boundary takes a row-by-row slow path that
// reloads (kept out of the unrolled fast loop, where it cost 12%).  Per row
// each pair of channels costs one packed multiply (factor * inv_rms) and one
// packed FMA (x * that + shift).  HBM traffic per row: x read, y written
// (2*D*esize bytes); with the residual h and branch read, h_out and y
// written (4*D*esize bytes, against 5*D*esize for the two ops apart).
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

// Widen the modulation of (sample, modality) `key` to fp32 for this
// thread's slots: fac = gamma * (1 + scale), sh = shift, gt = gate.
template <typename T, int NT, int VPT, bool RESID>
__device__ __forceinline__ void load_modulation(const RmsArgs &a, int key, int tid,
                                                const bool (&ok)[VPT],
                                                float2 (&fac)[VPT][Io<T>::E / 2],
                                                float2 (&sh)[VPT][Io<T>::E / 2],
                                                float2 (&gt)[RESID ? VPT : 1][Io<T>::E / 2]) {
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
      if constexpr (RESID)
        IO::unpack(ld_shared_vec(static_cast<const uint4 *>(a.gate) + koff + k * NT), gt[k]);
    }
  }
}

template <typename T, int NT, int VPT, int R, int S, bool RESID, int K = 0, bool FULL = false>
__global__ void __launch_bounds__(NT) rms_adaln_kernel(const RmsArgs a) {
  static_assert(K % R == 0, "an iteration's rows must lie in one chunk");
  using IO = Io<T>;
  constexpr int P = IO::E / 2;  // fp32 pairs per 16-byte vector
  constexpr int NW = NT / 32;
  constexpr int NIN = RESID ? 2 : 1;  // staged inputs per row: x, or h and branch
  extern __shared__ __align__(16) unsigned char smem[];
  float *red = reinterpret_cast<float *>(smem);                     // [2][R][32]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + 2 * R * 32 * 4);  // [S][R][NIN][VPT][NT]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;

  // slot k holds vector k*NT + tid of the row; FULL: the split covers the
  // row exactly, no access needs a guard
  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = FULL || k * NT + tid < a.nvec;

  for (int i = tid; i < 2 * R * 32; i += NT) red[i] = 0.f;  // unused warp slots read 0
  __syncthreads();

  RowOrder<K, R> ro;  // the CTA's rows, walked with local index j
  ro.init(a.rows);
  const int count = ro.count;
  const int iters = (count + R - 1) / R;
  const unsigned char *xc = static_cast<const unsigned char *>(a.x);
  const unsigned char *bc = RESID ? static_cast<const unsigned char *>(a.branch) : nullptr;
  unsigned char *yc = static_cast<unsigned char *>(a.y);
  unsigned char *hc = RESID ? static_cast<unsigned char *>(a.h_out) : nullptr;

  auto slot = [&](int s, int q, int in, int k) -> uint4 * {
    return &ring[(((s * R + q) * NIN + in) * VPT + k) * NT + tid];
  };
  // Copy this thread's slots of iteration `it`'s rows into ring stage s;
  // always commits a group (possibly empty) so the group count is uniform.
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
#pragma unroll
        for (int in = 0; in < NIN; ++in) {
          const uint4 *src =
              reinterpret_cast<const uint4 *>((in == 0 ? xc : bc) + ro.row(j) * row_bytes) + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k)
            if (ok[k]) cp_async16(slot(s, q, in, k), src + k * NT);
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);

  float2 fac[VPT][P], sh[VPT][P];  // gamma*(1+scale) and shift of `key`
  float2 gt[RESID ? VPT : 1][P];   // gate of `key` (residual only)
  int key = -1;                    // 2*b + m those belong to
  int cons = 0;                    // ring stage of iteration `it`
  int buf = 0;                     // which half of `red`
  TokenCursor cur;

  // Row q of the current stage into fp32 xq (with the residual: formed from
  // h and branch and written to h_out); returns this warp's sum of squares.
  auto load_row = [&](int q, int j, float2 (&xq)[VPT][P]) -> float {
    float2 acc = splat2(0.f);
    uint4 *hrow = RESID ? reinterpret_cast<uint4 *>(hc + ro.row(j) * row_bytes) + tid : nullptr;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (ok[k]) {
        IO::unpack(*slot(cons, q, 0, k), xq[k]);
        if constexpr (RESID) {
          float2 bq[P];
          IO::unpack(*slot(cons, q, 1, k), bq);
#pragma unroll
          for (int m = 0; m < P; ++m) xq[k][m] = fma2(gt[k][m], bq[m], xq[k][m]);
          st_stream16(hrow + k * NT, IO::pack(xq[k]));
        }
#pragma unroll
        for (int m = 0; m < P; ++m) acc = fma2(xq[k][m], xq[k][m], acc);
      }
    }
    return warp_sum(acc.x + acc.y);
  };
  // CTA total of the warp sums parked in red[buf][q] (after the barrier).
  auto cta_total = [&](int q) -> float {
    const float4 *r4 = reinterpret_cast<const float4 *>(red + (buf * R + q) * 32);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < (NW + 3) / 4; ++w) {
      const float4 v = r4[w];
      t += (v.x + v.y) + (v.z + v.w);
    }
    return t;
  };
  auto store_row = [&](int j, const float2 (&xq)[VPT][P], float tot) {
    const float2 inv2 = splat2(rsqrtf(fmaf(tot, a.inv_D, a.eps)));
    uint4 *yrow = reinterpret_cast<uint4 *>(yc + ro.row(j) * row_bytes) + tid;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      if (ok[k]) {
        float2 o[P];
#pragma unroll
        for (int m = 0; m < P; ++m) o[m] = fma2(xq[k][m], mul2(fac[k][m], inv2), sh[k][m]);
        st_stream16(yrow + k * NT, IO::pack(o));
      }
    }
  };

  for (int it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);
    if (ro.run_start(it * R)) cur.init(ro.row(it * R), a.L);
    const int nrows = count - it * R < R ? count - it * R : R;
    bool same = true;  // every row of this iteration uses the cached modulation
    {
      TokenCursor c = cur;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        if (q < nrows) same &= (2 * c.b + (c.r >= a.n_video ? 1 : 0)) == key;
        c.next(a.L);
      }
    }
    cp_async_wait<S - 1>();

    if (same) {
      float2 xp[R][VPT][P];
      float tot[R];
#pragma unroll
      for (int q = 0; q < R; ++q) tot[q] = q < nrows ? load_row(q, it * R + q, xp[q]) : 0.f;
      if (NW > 1) {
        if (lane == 0) {
#pragma unroll
          for (int q = 0; q < R; ++q) red[(buf * R + q) * 32 + warp] = tot[q];
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < R; ++q) tot[q] = cta_total(q);
      }
#pragma unroll
      for (int q = 0; q < R; ++q)
        if (q < nrows) store_row(it * R + q, xp[q], tot[q]);
#pragma unroll
      for (int q = 0; q < R; ++q)
        if (q < nrows) cur.next(a.L);
    } else {
      // A modality or sample boundary falls in this iteration: reload the
      // modulation row by row (at most a few times per CTA), one barrier per row.
#pragma unroll 1
      for (int q = 0; q < nrows; ++q) {
        const int nkey = 2 * cur.b + (cur.r >= a.n_video ? 1 : 0);
        if (nkey != key) {
          key = nkey;
          load_modulation<T, NT, VPT, RESID>(a, key, tid, ok, fac, sh, gt);
        }
        float2 xq[VPT][P];
        float tot = load_row(q, it * R + q, xq);
        if (NW > 1) {
          if (lane == 0) red[(buf * R + q) * 32 + warp] = tot;
          __syncthreads();
          tot = cta_total(q);
        }
        store_row(it * R + q, xq, tot);
        cur.next(a.L);
      }
    }
    buf ^= 1;
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

// Two rows per iteration while the registers allow it (the residual keeps a
// third fp32 modulation vector, the gate, resident).
template <int VPT, bool RESID>
constexpr int kRows = VPT <= (RESID ? 3 : 5) ? 2 : 1;

// Rows go to the CTAs in chunks of kRmsChunk dealt round-robin, so the grid
// works through one contiguous window of the tensors: 0.398 against
// 0.416 ms for a contiguous share per CTA (RMS-AdaLN at the 5 s clip, output
// bit-identical), 0.820 against 0.839 ms with the residual.
constexpr int kRmsChunk = 8;

template <typename T, int NT, int VPT, bool RESID, bool FULL, int R = kRows<VPT, RESID>,
          int S = 2, int K = kRmsChunk>
cudaError_t launch_t(const RmsArgs &a, cudaStream_t stream, Geometry *geo) {
  constexpr int NIN = RESID ? 2 : 1;
  if (FULL && a.nvec != NT * VPT) return cudaErrorInvalidValue;
  const void *fn =
      reinterpret_cast<const void *>(&rms_adaln_kernel<T, NT, VPT, R, S, RESID, K, FULL>);
  const size_t smem = 2 * R * 32 * 4 + static_cast<size_t>(S) * R * NIN * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  rms_adaln_kernel<T, NT, VPT, R, S, RESID, K, FULL>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

// A short launch whose split covers the row exactly (128 x 5 at D = 5120)
// takes the unguarded instantiation (FULL): at 8,264 rows it streams 5.5
// instead of 4.35 TB/s.  Longer launches keep the guards, which measured
// 3-4% faster there (126,552 and 371,592 rows, two boxes, four bench runs
// each way); the results are bit-identical either way.
constexpr int64_t kFullMaxRows = 16384;

template <typename T, bool RESID>
cudaError_t dispatch(const RmsArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
#define SOL_CASE(NT, V)                                                       \
  if (threads == NT && vpt == V)                                              \
    return a.nvec == NT * V && a.rows <= kFullMaxRows                         \
               ? launch_t<T, NT, V, RESID, true>(a, stream, geo)              \
               : launch_t<T, NT, V, RESID, false>(a, stream, geo);
  SOL_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

template <bool RESID>
cudaError_t launch_any(const RmsArgs &a, int dtype, cudaStream_t stream, Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!pick_split(a.nvec, &threads, &vpt)) return cudaErrorInvalidValue;
  return dtype == 0 ? dispatch<float, RESID>(a, threads, vpt, stream, geo)
                    : dispatch<__nv_bfloat16, RESID>(a, threads, vpt, stream, geo);
}

}  // namespace

cudaError_t launch_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream, Geometry *geo) {
  return launch_any<false>(a, dtype, stream, geo);
}

cudaError_t launch_gate_residual_rms_adaln(const RmsArgs &a, int dtype, cudaStream_t stream,
                                           Geometry *geo) {
  return launch_any<true>(a, dtype, stream, geo);
}

}  // namespace sol
