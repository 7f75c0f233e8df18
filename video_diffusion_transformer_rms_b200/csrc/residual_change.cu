// First-Block-Cache change detector (Sol Video Inference Engine MiniMax-H3
// page, cross-step caching paragraph: the first transformer block's residual
// is the proxy for the whole stack, and the remaining blocks are skipped when
// it has barely moved since the previous step, against one threshold).
//
// For each sample b of [B, L, D] residuals and for the whole batch:
//   num = sum |cur - prev|,  den = sum |prev|,  rel = num / den
// and, optionally, prev_out = cur (the cache refresh) in the same pass.
//
// Grid: blockIdx.y = sample, blockIdx.x = one of `ctas_per_sample` CTAs
// that split the sample's rows into contiguous shares, so a CTA never mixes
// samples.  Rows stream HBM -> shared memory through the same cp.async ring
// as the normalisation kernels (cur and prev side by side).  Each thread sums
// a row's |differences| in fp32 (at most 8 vectors of 8 elements) and adds
// the row total to fp64 accumulators; the CTA reduces its threads in a fixed
// order and writes (num, den) to its own workspace slot.  A one-CTA finalize
// kernel then sums the slots of each sample in a fixed order, so the result
// is deterministic: no atomics, and no workspace state survives between
// calls (every slot is rewritten on every call).  HBM traffic per row:
// 2*D*esize bytes read, plus D*esize written with the cache refresh.
#include <math.h>

#include <map>
#include <mutex>

#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

constexpr int kFinalThreads = 256;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T, int NT, int VPT, int R, int S, bool COPY>
__global__ void __launch_bounds__(NT) residual_change_kernel(const ChangeArgs a) {
  using IO = Io<T>;
  constexpr int P = IO::E / 2;
  constexpr int NW = NT / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  double *red = reinterpret_cast<double *>(smem);                    // [NW][2]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + 32 * 2 * 8);       // [S][R][2][VPT][NT]

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int b = blockIdx.y;
  const int64_t row_bytes = static_cast<int64_t>(a.nvec) * 16;

  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = k * NT + tid < a.nvec;

  int64_t begin;
  int count;
  cta_rows(a.L, blockIdx.x, gridDim.x, begin, count);
  begin += static_cast<int64_t>(b) * a.L;
  const int iters = (count + R - 1) / R;
  const unsigned char *cc = static_cast<const unsigned char *>(a.cur) + begin * row_bytes;
  const unsigned char *pc = static_cast<const unsigned char *>(a.prev) + begin * row_bytes;
  unsigned char *oc = COPY ? static_cast<unsigned char *>(a.prev_out) + begin * row_bytes : nullptr;

  auto slot = [&](int s, int q, int in, int k) -> uint4 * {
    return &ring[(((s * R + q) * 2 + in) * VPT + k) * NT + tid];
  };
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const uint4 *cs = reinterpret_cast<const uint4 *>(cc + j * row_bytes) + tid;
        const uint4 *ps = reinterpret_cast<const uint4 *>(pc + j * row_bytes) + tid;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            cp_async16(slot(s, q, 0, k), cs + k * NT);
            cp_async16(slot(s, q, 1, k), ps + k * NT);
          }
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);

  double num = 0.0, den = 0.0;
  int cons = 0;
  for (int it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);
    cp_async_wait<S - 1>();
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        float n0 = 0.f, n1 = 0.f, d0 = 0.f, d1 = 0.f;
        uint4 *orow = COPY ? reinterpret_cast<uint4 *>(oc + j * row_bytes) + tid : nullptr;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
          if (ok[k]) {
            const uint4 craw = *slot(cons, q, 0, k);
            float2 cv[P], pv[P];
            IO::unpack(craw, cv);
            IO::unpack(*slot(cons, q, 1, k), pv);
#pragma unroll
            for (int m = 0; m < P; ++m) {
              n0 += fabsf(cv[m].x - pv[m].x);
              n1 += fabsf(cv[m].y - pv[m].y);
              d0 += fabsf(pv[m].x);
              d1 += fabsf(pv[m].y);
            }
            if constexpr (COPY) st_stream16(orow + k * NT, craw);
          }
        }
        num += static_cast<double>(n0 + n1);
        den += static_cast<double>(d0 + d1);
      }
    }
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();

  num = warp_sum_d(num);
  den = warp_sum_d(den);
  if (lane == 0) {
    red[warp * 2 + 0] = num;
    red[warp * 2 + 1] = den;
  }
  __syncthreads();
  if (tid == 0) {
    double tn = 0.0, td = 0.0;
    for (int w = 0; w < NW; ++w) {
      tn += red[w * 2 + 0];
      td += red[w * 2 + 1];
    }
    double *slot_out = a.partial + (static_cast<int64_t>(b) * kMaxChangeCtas + blockIdx.x) * 2;
    slot_out[0] = tn;
    slot_out[1] = td;
  }
}

// One CTA: per sample, the fixed-order sum of its CTAs' slots; then the batch.
__global__ void __launch_bounds__(kFinalThreads) residual_change_finalize(const ChangeArgs a) {
  __shared__ double red[kFinalThreads / 32][2];
  const int tid = threadIdx.x;
  double bn = 0.0, bd = 0.0;  // batch totals (thread 0)
  for (int b = 0; b < a.B; ++b) {
    const double *p = a.partial + static_cast<int64_t>(b) * kMaxChangeCtas * 2;
    double n = 0.0, d = 0.0;
    for (int i = tid; i < a.ctas_per_sample; i += kFinalThreads) {
      n += p[2 * i + 0];
      d += p[2 * i + 1];
    }
    n = warp_sum_d(n);
    d = warp_sum_d(d);
    if ((tid & 31) == 0) {
      red[tid >> 5][0] = n;
      red[tid >> 5][1] = d;
    }
    __syncthreads();
    if (tid == 0) {
      double tn = 0.0, td = 0.0;
      for (int w = 0; w < kFinalThreads / 32; ++w) {
        tn += red[w][0];
        td += red[w][1];
      }
      a.out[3 * b + 0] = tn;
      a.out[3 * b + 1] = td;
      a.out[3 * b + 2] = td > 0.0 ? tn / td : (tn > 0.0 ? static_cast<double>(INFINITY) : 0.0);
      bn += tn;
      bd += td;
    }
    __syncthreads();
  }
  if (tid == 0) {
    a.out[3 * a.B + 0] = bn;
    a.out[3 * a.B + 1] = bd;
    a.out[3 * a.B + 2] = bd > 0.0 ? bn / bd : (bn > 0.0 ? static_cast<double>(INFINITY) : 0.0);
  }
}

template <typename T, int NT, int VPT, bool COPY>
cudaError_t launch_t(ChangeArgs a, cudaStream_t stream, Geometry *geo) {
  constexpr int R = VPT <= 6 ? 2 : 1;
  constexpr int S = 2;
  const void *fn = reinterpret_cast<const void *>(&residual_change_kernel<T, NT, VPT, R, S, COPY>);
  const size_t smem = 32 * 2 * 8 + static_cast<size_t>(S) * R * 2 * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t per_sample = (static_cast<int64_t>(per_sm) * device_sms() + a.B - 1) / a.B;
  if (per_sample > a.L) per_sample = a.L;
  if (per_sample > kMaxChangeCtas) per_sample = kMaxChangeCtas;
  if (per_sample < 1) per_sample = 1;
  a.ctas_per_sample = static_cast<int>(per_sample);
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(per_sample * a.B)};
  const dim3 grid(static_cast<unsigned>(per_sample), static_cast<unsigned>(a.B));
  residual_change_kernel<T, NT, VPT, R, S, COPY><<<grid, NT, smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  residual_change_finalize<<<1, kFinalThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

template <typename T, bool COPY>
cudaError_t dispatch(const ChangeArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch_t<T, NT, V, COPY>(a, stream, geo);
  SOL_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_residual_change(const ChangeArgs &a, int dtype, cudaStream_t stream,
                                   Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!pick_split(a.nvec, &threads, &vpt)) return cudaErrorInvalidValue;
  const bool copy = a.prev_out != nullptr;
  if (dtype == 0)
    return copy ? dispatch<float, true>(a, threads, vpt, stream, geo)
                : dispatch<float, false>(a, threads, vpt, stream, geo);
  return copy ? dispatch<__nv_bfloat16, true>(a, threads, vpt, stream, geo)
              : dispatch<__nv_bfloat16, false>(a, threads, vpt, stream, geo);
}

// ---------------------------------------------------------------------------
// Variant for callers that cannot allocate device memory: the partial sums go
// to this file-scope array instead of a caller workspace.  It is sized for
// kNoAllocMaxSamples samples (256 KiB) and every device that loads the
// library holds it until the process exits.  Host code must not pass the
// symbol itself to a kernel (in host code it is only a stand-in): the device
// address is looked up with cudaGetSymbolAddress, once per device, with that
// device current, on the first call made on it.
// ---------------------------------------------------------------------------
static __device__ __align__(256) double g_change_scratch[kNoAllocMaxSamples * kMaxChangeCtas * 2];

namespace {

cudaError_t noalloc_scratch(double **ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::mutex mu;
  static std::map<int, double *> addr;
  std::lock_guard<std::mutex> lk(mu);
  auto it = addr.find(dev);
  if (it == addr.end()) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_change_scratch);
    if (e != cudaSuccess) return e;
    it = addr.emplace(dev, static_cast<double *>(p)).first;
  }
  *ptr = it->second;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_residual_change_noalloc(ChangeArgs a, int dtype, cudaStream_t stream,
                                           Geometry *geo) {
  if (a.B > kNoAllocMaxSamples) return cudaErrorInvalidValue;
  double *scratch = nullptr;
  cudaError_t e = noalloc_scratch(&scratch);
  if (e != cudaSuccess) return e;
  a.partial = scratch;
  return launch_residual_change(a, dtype, stream, geo);
}

}  // namespace sol
