// AdaLN-gated residual add: out = h + gate[b][m] * branch per token row
// (the gate of the adaLN DiT block; one of the elementwise chains the Sol
// Video Inference Engine MiniMax-H3 page removes by fusion).
//
// Same persistent cp.async ring as RMS-AdaLN (round-robin chunks of rows per
// CTA, R rows per iteration, compile-time CTA size and vectors per thread),
// with h and branch staged side by side and no reduction; one CTA barrier
// per iteration keeps the warps together.  The gate vector of the current (sample, modality) is widened to
// fp32 registers only when the CTA crosses a modality or sample boundary;
// per row each pair of channels is one packed fp32x2 FMA.  HBM traffic:
// read h, read branch, write out = 3*D*esize bytes per row.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

template <typename T, int NT, int VPT, int R, int S, int K = 0, bool BAR = false,
          bool FULL = false>
__global__ void __launch_bounds__(NT) gate_residual_kernel(const GateArgs a) {
  static_assert(K % R == 0, "an iteration's rows must lie in one chunk");
  using IO = Io<T>;
  constexpr int P = IO::E / 2;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4 *ring = reinterpret_cast<uint4 *>(smem);  // [S][R][2][VPT][NT]

  const int tid = threadIdx.x;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;
  const unsigned char *hb = static_cast<const unsigned char *>(a.h);
  const unsigned char *bb = static_cast<const unsigned char *>(a.branch);
  unsigned char *ob = static_cast<unsigned char *>(a.out);

  // FULL: the split covers the row exactly, no access needs a guard
  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = FULL || k * NT + tid < a.nvec;

  RowOrder<K, R> ro;
  ro.init(a.rows);
  const int count = ro.count;
  const int iters = (count + R - 1) / R;
  auto slot = [&](int s, int q, int which, int k) -> uint4 * {
    return &ring[(((s * R + q) * 2 + which) * VPT + k) * NT + tid];
  };
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const int64_t off = ro.row(j) * row_bytes;
        const uint4 *hs = reinterpret_cast<const uint4 *>(hb + off) + tid;
        const uint4 *bs = reinterpret_cast<const uint4 *>(bb + off) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            cp_async16(slot(s, q, 0, k), hs + k * NT);
            cp_async16(slot(s, q, 1, k), bs + k * NT);
          }
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);

  float2 gv[VPT][P];
  int key = -1;
  int cons = 0;
  TokenCursor cur;
  for (int it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);
    if (ro.run_start(it * R)) cur.init(ro.row(it * R), a.L);
    cp_async_wait<S - 1>();
    if constexpr (BAR) __syncthreads();  // the CTA's warps on the same rows
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const int nkey = 2 * cur.b + (cur.r >= a.n_video ? 1 : 0);
        if (nkey != key) {
          key = nkey;
          const uint4 *g0 =
              static_cast<const uint4 *>(a.gate) + static_cast<int64_t>(key) * a.nvec + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k)
            if (ok[k]) IO::unpack(ld_shared_vec(g0 + k * NT), gv[k]);
        }
        uint4 *orow = reinterpret_cast<uint4 *>(ob + ro.row(j) * row_bytes) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            float2 hf[P], bf[P], o[P];
            IO::unpack(*slot(cons, q, 0, k), hf);
            IO::unpack(*slot(cons, q, 1, k), bf);
#pragma unroll
            for (int m = 0; m < P; ++m) o[m] = fma2(gv[k][m], bf[m], hf[m]);
            st_stream16(orow + k * NT, IO::pack(o));
          }
        }
        cur.next(a.L);
      }
    }
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

// Rows in chunks of kGateChunk dealt round-robin over the CTAs (the grid sweeps
// one contiguous window), with a CTA barrier per iteration although nothing
// is shared: it keeps the CTA's warps on the same rows.  0.605 against
// 0.633 ms for a contiguous share per CTA without the barrier (5 s clip).
constexpr int kGateChunk = 8;

template <typename T, int NT, int VPT, bool FULL, int R = (VPT <= 6 ? 2 : 1), int S = 2,
          int K = kGateChunk, bool BAR = true>
cudaError_t launch_t(const GateArgs &a, cudaStream_t stream, Geometry *geo) {
  if (FULL && a.nvec != NT * VPT) return cudaErrorInvalidValue;
  const void *fn =
      reinterpret_cast<const void *>(&gate_residual_kernel<T, NT, VPT, R, S, K, BAR, FULL>);
  const size_t smem = static_cast<size_t>(S) * R * 2 * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  gate_residual_kernel<T, NT, VPT, R, S, K, BAR, FULL>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

// A split that covers the row exactly (128 x 5 at D = 5120) takes the
// unguarded instantiation (FULL): 0.607 -> 0.598 ms at the 5 s clip in one
// interleaved session, bit-identical.
template <typename T>
cudaError_t dispatch(const GateArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
#define SOL_CASE(NT, V)                                                 \
  if (threads == NT && vpt == V)                                        \
    return a.nvec == NT * V ? launch_t<T, NT, V, true>(a, stream, geo)  \
                            : launch_t<T, NT, V, false>(a, stream, geo);
  SOL_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gate_residual(const GateArgs &a, int dtype, cudaStream_t stream,
                                 Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!pick_split(a.nvec, &threads, &vpt)) return cudaErrorInvalidValue;
  return dtype == 0 ? dispatch<float>(a, threads, vpt, stream, geo)
                    : dispatch<__nv_bfloat16>(a, threads, vpt, stream, geo);
}

}  // namespace sol
