// Fused per-head QKNorm + 3D multimodal RoPE on a merged QKV projection
// (Sol Video Inference Engine MiniMax-H3 page, fusion table, rows "fused
// QKNorm + RoPE" and "QKV merge"; rotary embedding of RoFormer with the
// frequency list split into t / h / w sections).
//
// Per token row: q = columns [0, D), k = [D, 2D) of the merged row; every
// head (head_dim channels) is RMS-normalised in fp32, scaled by gamma_q or
// gamma_k, and its adjacent pairs (2i, 2i+1) are rotated by
// pos_axis(i) * theta^(-2i/head_dim).  v is never touched.
//
// Work split: a CTA streams whole rows (q and k: 2*D*esize bytes) through a
// cp.async ring.  G = head_dim*esize/16 consecutive lanes own one head, so a
// head's sum of squares is G-lane shuffles, no shared memory.  Because the
// CTA size is a multiple of G, a thread always sees the same lane-in-head,
// hence the same rotary pairs and gamma entries, in every head it visits.
// The 64 (cos, sin) values of a row are shared by all 2*n_heads head vectors
// of the row: the CTA computes them once per row (angle reduced modulo 2*pi
// in fp64, then sincosf on the reduced fp32 angle, accurate for positions in
// the thousands) into a double-buffered shared table.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

constexpr int kMaxV = 8;          // 16-byte vectors per thread per row
constexpr int kMaxPairs = 128;    // head_dim <= 256
constexpr size_t kHeader = 3072;  // freq[128] double + cos[2][128] + sin[2][128] float
constexpr double k2Pi = 6.283185307179586476925286766559;
constexpr double kInv2Pi = 0.15915494309189533576888376337251;

template <typename T, int G, int S>
__global__ void __launch_bounds__(kMaxThreads)
    qknorm_rope3d_kernel(const QkArgs a, const int vpt) {
  using IO = Io<T>;
  constexpr int E = IO::E;
  constexpr int PPV = E / 2;  // rotary pairs per 16-byte vector
  extern __shared__ __align__(16) unsigned char smem[];
  double *freq = reinterpret_cast<double *>(smem);
  float *cosb = reinterpret_cast<float *>(smem + 1024);   // [2][kMaxPairs]
  float *sinb = reinterpret_cast<float *>(smem + 2048);   // [2][kMaxPairs]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + kHeader);  // [S][vpt][threads]

  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int gl = tid % G;    // lane within the head
  const int p0 = gl * PPV;   // first rotary pair of this thread's slot
  const int64_t step = gridDim.x;
  const unsigned char *qkv = static_cast<const unsigned char *>(a.qkv);
  unsigned char *qo = static_cast<unsigned char *>(a.q_out);
  unsigned char *ko = static_cast<unsigned char *>(a.k_out);

  float gq[E], gk[E];
  if (a.gamma_q) {
    IO::unpack(ld_shared_vec(static_cast<const uint4 *>(a.gamma_q) + gl), gq);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) gq[e] = 1.f;
  }
  if (a.gamma_k) {
    IO::unpack(ld_shared_vec(static_cast<const uint4 *>(a.gamma_k) + gl), gk);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) gk[e] = 1.f;
  }
  for (int p = tid; p < a.npairs; p += nt)
    freq[p] = pow(static_cast<double>(a.theta), -2.0 * p / a.head_dim);

  auto issue = [&](int64_t r, int s) {
    if (r < a.rows) {
      const uint4 *src = reinterpret_cast<const uint4 *>(qkv + r * a.ld_qkv_bytes);
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
  __syncthreads();  // freq[] visible

  int cons = 0;
  int buf = 0;
  for (; row < a.rows; row += step) {
    issue(row + (S - 1) * step, cons == 0 ? S - 1 : cons - 1);

    // rotary angles of this row
    const int64_t b = row / a.L;
    const int64_t r = row - b * a.L;
    int64_t pt, ph, pw;
    if (r < a.n_video) {
      pt = r / a.HW;
      const int64_t rem = r - pt * a.HW;
      ph = rem / a.W;
      pw = rem - ph * a.W;
    } else {
      pt = r - a.n_video;
      ph = 0;
      pw = 0;
    }
    for (int p = tid; p < a.npairs; p += nt) {
      const int64_t pos = p < a.sec_t ? pt : (p < a.sec_th ? ph : pw);
      const double ang = static_cast<double>(pos) * freq[p];
      const double turns = rint(ang * kInv2Pi);
      const float red = static_cast<float>(fma(-turns, k2Pi, ang));
      float sv, cv;
      sincosf(red, &sv, &cv);
      cosb[buf * kMaxPairs + p] = cv;
      sinb[buf * kMaxPairs + p] = sv;
    }

    cp_async_wait<S - 1>();
    __syncthreads();  // angle table of this row visible

    float cs[PPV], sn[PPV];
#pragma unroll
    for (int j = 0; j < PPV; ++j) {
      cs[j] = cosb[buf * kMaxPairs + p0 + j];
      sn[j] = sinb[buf * kMaxPairs + p0 + j];
    }

#pragma unroll
    for (int k = 0; k < kMaxV; ++k) {
      if (k < vpt) {  // uniform over the CTA: every lane joins the shuffles
        const int v = k * nt + tid;
        const bool valid = v < a.nvec;  // uniform over each head's G lanes
        uint4 xv = make_uint4(0u, 0u, 0u, 0u);
        if (valid) xv = ring[(cons * vpt + k) * nt + tid];
        float f[E];
        IO::unpack(xv, f);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(f[e], f[e], ss);
        ss = group_sum<G>(ss);
        const float inv = rsqrtf(fmaf(ss, a.inv_hd, a.eps));
        const bool is_k = v >= a.nvec_q;
        float o[E];
#pragma unroll
        for (int j = 0; j < PPV; ++j) {
          const float x0 = f[2 * j] * inv * (is_k ? gk[2 * j] : gq[2 * j]);
          const float x1 = f[2 * j + 1] * inv * (is_k ? gk[2 * j + 1] : gq[2 * j + 1]);
          o[2 * j] = fmaf(x0, cs[j], -x1 * sn[j]);
          o[2 * j + 1] = fmaf(x0, sn[j], x1 * cs[j]);
        }
        if (valid) {
          unsigned char *dst =
              is_k ? ko + row * a.ld_out_bytes + static_cast<int64_t>(v - a.nvec_q) * 16
                   : qo + row * a.ld_out_bytes + static_cast<int64_t>(v) * 16;
          st_stream16(dst, IO::pack(o));
        }
      }
    }
    buf ^= 1;
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <typename T, int G, int S>
cudaError_t launch_t(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  const void *fn = reinterpret_cast<const void *>(&qknorm_rope3d_kernel<T, G, S>);
  const size_t smem = kHeader + static_cast<size_t>(S) * vpt * threads * 16;
  const int per_sm = resident_blocks(fn, threads, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{threads, vpt, S, smem, static_cast<int>(grid)};
  qknorm_rope3d_kernel<T, G, S><<<static_cast<unsigned>(grid), threads, smem, stream>>>(a, vpt);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t launch_s(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  const size_t stage = static_cast<size_t>(vpt) * threads * 16;
  if (stage <= 24 * 1024) return launch_t<T, G, 3>(a, threads, vpt, stream, geo);
  return launch_t<T, G, 2>(a, threads, vpt, stream, geo);
}

template <typename T>
cudaError_t launch_g(const QkArgs &a, int G, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
  switch (G) {
    case 2: return launch_s<T, 2>(a, threads, vpt, stream, geo);
    case 4: return launch_s<T, 4>(a, threads, vpt, stream, geo);
    case 8: return launch_s<T, 8>(a, threads, vpt, stream, geo);
    case 16: return launch_s<T, 16>(a, threads, vpt, stream, geo);
    case 32: return launch_s<T, 32>(a, threads, vpt, stream, geo);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_qknorm_rope3d(const QkArgs &a, int dtype, cudaStream_t stream,
                                 Geometry *geo) {
  const int esize = dtype == 0 ? 4 : 2;
  const int G = a.head_dim * esize / 16;  // lanes per head
  if (a.npairs > kMaxPairs) return cudaErrorInvalidValue;
  int threads = 0, vpt = 0;
  if (!row_split(a.nvec, 4, kMaxV, kMaxThreads, 32, &threads, &vpt)) return cudaErrorInvalidValue;
  return dtype == 0 ? launch_g<float>(a, G, threads, vpt, stream, geo)
                    : launch_g<__nv_bfloat16>(a, G, threads, vpt, stream, geo);
}

}  // namespace sol
