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
// Work split: a CTA streams its own contiguous share of the rows (q and k:
// 2*D*esize bytes each), R rows per iteration, through a cp.async ring and
// walks the rows' (t, h, w) positions incrementally.  G = head_dim*esize/16 consecutive lanes own one
// head, so a head's sum of squares is G-lane shuffles, no shared memory.  Because the
// CTA size is a multiple of G, a thread always sees the same lane-in-head,
// hence the same rotary pairs and gamma entries, in every head it visits.
// The 64 (cos, sin) values of a row are shared by all 2*n_heads head vectors
// of the row: the CTA computes them once per row (angle reduced modulo 2*pi
// in fp64, then sincosf on the reduced fp32 angle, accurate for positions in
// the thousands) into a double-buffered shared table, one barrier per R rows.  Pairs are processed
// two at a time with packed fp32x2 arithmetic (even and odd elements of two
// adjacent rotary pairs side by side), gamma folded into the rotation.
#pragma once
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace qk {

constexpr int kMaxPairs = 128;  // head_dim <= 256
constexpr double k2Pi = 6.283185307179586476925286766559;
constexpr double kInv2Pi = 0.15915494309189533576888376337251;

// Shared-memory header: freq[kMaxPairs] (fp64), then cos and sin tables
// [2 buffers][R rows][kMaxPairs] (fp32).
template <int R>
__host__ __device__ constexpr size_t header_bytes() {
  return kMaxPairs * 8 + 2 * (2 * R * kMaxPairs * 4);
}

template <typename T, int G, int NT, int VPT, int R, int S>
__global__ void __launch_bounds__(NT) qknorm_rope3d_kernel(const QkArgs a) {
  using IO = Io<T>;
  constexpr int E = IO::E;
  constexpr int PPV = E / 2;  // rotary pairs per 16-byte vector
  constexpr int Q = PPV / 2;  // float2 lanes of (pair 2m, pair 2m+1) per vector
  constexpr int TAB = 2 * R * kMaxPairs;
  extern __shared__ __align__(16) unsigned char smem[];
  double *freq = reinterpret_cast<double *>(smem);
  float *cosb = reinterpret_cast<float *>(smem + kMaxPairs * 8);         // [2][R][kMaxPairs]
  float *sinb = cosb + TAB;                                              // [2][R][kMaxPairs]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + header_bytes<R>());     // [S][R][2][VPT][NT]

  const int tid = threadIdx.x;
  const int gl = tid % G;   // lane within the head
  const int p0 = gl * PPV;  // first rotary pair of this thread's slot
  const unsigned char *qkv = static_cast<const unsigned char *>(a.qkv);
  unsigned char *qo = static_cast<unsigned char *>(a.q_out);
  unsigned char *ko = static_cast<unsigned char *>(a.k_out);
  const int64_t part_bytes = static_cast<int64_t>(a.nvec_q) * 16;

  bool ok[VPT];  // uniform over each head's G lanes (nvec_q and NT are multiples of G)
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = k * NT + tid < a.nvec_q;

  // gamma of this thread's slot in rotary layout (the same in every head):
  // gev[part][m] = (g[4m], g[4m+2]), god[part][m] = (g[4m+1], g[4m+3])
  float2 gev[2][Q], god[2][Q];
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const void *g = part == 0 ? a.gamma_q : a.gamma_k;
    if (g) {
      IO::unpack_eo(ld_shared_vec(static_cast<const uint4 *>(g) + gl), gev[part], god[part]);
    } else {
#pragma unroll
      for (int m = 0; m < Q; ++m) gev[part][m] = god[part][m] = splat2(1.f);
    }
  }
  for (int p = tid; p < a.npairs; p += NT)
    freq[p] = pow(static_cast<double>(a.theta), -2.0 * p / a.head_dim);

  int64_t begin;
  int count;
  cta_rows(a.rows, blockIdx.x, gridDim.x, begin, count);
  const int iters = (count + R - 1) / R;
  const unsigned char *src_c = qkv + begin * a.ld_qkv_bytes;
  unsigned char *qo_c = qo + begin * a.ld_out_bytes;
  unsigned char *ko_c = ko + begin * a.ld_out_bytes;
  auto slot = [&](int s, int q, int part, int k) -> uint4 * {
    return &ring[(((s * R + q) * 2 + part) * VPT + k) * NT + tid];
  };
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const unsigned char *src = src_c + j * a.ld_qkv_bytes;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint4 *ps = reinterpret_cast<const uint4 *>(src + part * part_bytes) + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k)
            if (ok[k]) cp_async16(slot(s, q, part, k), ps + k * NT);
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);
  __syncthreads();  // freq[] visible

  TokenCursor tok;
  tok.init(begin, a.L);
  GridCursor pos;
  pos.init(tok.r, a.n_video, a.HW, a.W);
  int cons = 0;
  int buf = 0;
  for (int it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);

    // positions of this iteration's rows (rows past `end` are never read)
    int pt[R], ph[R], pw[R];
    {
      TokenCursor t2 = tok;
      GridCursor g2 = pos;
#pragma unroll
      for (int q = 0; q < R; ++q) {
        pt[q] = g2.t;
        ph[q] = g2.h;
        pw[q] = g2.w;
        t2.next(a.L);
        g2.next(t2.r, a.n_video, a.H, a.W);
      }
    }
    // (cos, sin) of every row's rotary angles, angle reduced modulo 2*pi in fp64
    for (int idx = tid; idx < R * a.npairs; idx += NT) {
      int q = 0, p = idx;
#pragma unroll
      for (int qq = 1; qq < R; ++qq)
        if (p >= a.npairs) {
          p -= a.npairs;
          q = qq;
        }
      int at = pw[0];
#pragma unroll
      for (int qq = 0; qq < R; ++qq)
        if (q == qq) at = p < a.sec_t ? pt[qq] : (p < a.sec_th ? ph[qq] : pw[qq]);
      const double ang = static_cast<double>(at) * freq[p];
      const double turns = rint(ang * kInv2Pi);
      const float red = static_cast<float>(fma(-turns, k2Pi, ang));
      float sv, cv;
      sincosf(red, &sv, &cv);
      cosb[(buf * R + q) * kMaxPairs + p] = cv;
      sinb[(buf * R + q) * kMaxPairs + p] = sv;
    }

    cp_async_wait<S - 1>();
    __syncthreads();  // angle tables of these rows visible

#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        // cs[m] = (cos of pair p0+2m, cos of pair p0+2m+1); likewise sn
        float2 cs[Q], sn[Q];
#pragma unroll
        for (int m = 0; m < Q; ++m) {
          cs[m] = *reinterpret_cast<const float2 *>(&cosb[(buf * R + q) * kMaxPairs + p0 + 2 * m]);
          sn[m] = *reinterpret_cast<const float2 *>(&sinb[(buf * R + q) * kMaxPairs + p0 + 2 * m]);
        }
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          // gamma folded into the rotation of each pair (x0, x1):
          //   u0 = x0*(g0 c) + x1*(-g1 s),  u1 = x0*(g0 s) + x1*(g1 c),  out = inv*u
          float2 c0[Q], ns1[Q], s0[Q], c1[Q];
#pragma unroll
          for (int m = 0; m < Q; ++m) {
            c0[m] = mul2(gev[part][m], cs[m]);
            s0[m] = mul2(gev[part][m], sn[m]);
            ns1[m] = mul2(god[part][m], make_float2(-sn[m].x, -sn[m].y));
            c1[m] = mul2(god[part][m], cs[m]);
          }
          uint4 *dst =
              reinterpret_cast<uint4 *>((part == 0 ? qo_c : ko_c) + j * a.ld_out_bytes) + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            // every lane joins the shuffles; ok[] only guards memory accesses
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (ok[k]) xv = *slot(cons, q, part, k);
            float2 ev[Q], od[Q];
            IO::unpack_eo(xv, ev, od);
            float2 acc = mul2(ev[0], ev[0]);
            acc = fma2(od[0], od[0], acc);
#pragma unroll
            for (int m = 1; m < Q; ++m) {
              acc = fma2(ev[m], ev[m], acc);
              acc = fma2(od[m], od[m], acc);
            }
            const float ss = group_sum<G>(acc.x + acc.y);
            const float2 inv2 = splat2(rsqrtf(fmaf(ss, a.inv_hd, a.eps)));
            float2 u0[Q], u1[Q];
#pragma unroll
            for (int m = 0; m < Q; ++m) {
              u0[m] = mul2(fma2(od[m], ns1[m], mul2(ev[m], c0[m])), inv2);
              u1[m] = mul2(fma2(od[m], c1[m], mul2(ev[m], s0[m])), inv2);
            }
            if (ok[k]) st_stream16(dst + k * NT, IO::pack_eo(u0, u1));
          }
        }
        tok.next(a.L);
        pos.next(tok.r, a.n_video, a.H, a.W);
      }
    }
    buf ^= 1;
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <typename T, int G, int NT, int VPT>
cudaError_t launch(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  constexpr int R = VPT <= 6 ? 2 : 1;  // keeps the ring within shared memory
  constexpr int S = 2;
  const void *fn = reinterpret_cast<const void *>(&qknorm_rope3d_kernel<T, G, NT, VPT, R, S>);
  const size_t smem = header_bytes<R>() + static_cast<size_t>(S) * R * 2 * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  qknorm_rope3d_kernel<T, G, NT, VPT, R, S>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

template <typename T, int G>
cudaError_t dispatch(const QkArgs &a, int threads, int vpt, cudaStream_t stream, Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch<T, G, NT, V>(a, stream, geo);
  SOL_QK_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace qk
}  // namespace sol
