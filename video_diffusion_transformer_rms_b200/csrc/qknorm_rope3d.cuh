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
//
// Table-driven form (TAB): the caller builds a rotary table once per
// (positions, theta, head_dim, sections) -- row p holds cos(p*f_i) for every
// pair i, then sin(p*f_i), each computed in fp64 and rounded once to fp32 --
// and every thread reads the (cos, sin) of its own pairs at the row's
// position on their axis straight from it (read-only path; the table is a few
// hundred KB to a few MB and stays in L1/L2).  That removes the per-row fp64
// angle work, sincosf, the shared angle tables and the CTA barrier: no thread
// of the CTA waits for another, and the ring can run deeper.
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

// Rotary axis of pair p: 0 = t, 1 = h, 2 = w.
__device__ __forceinline__ int pair_axis(int p, int sec_t, int sec_th) {
  return p < sec_t ? 0 : (p < sec_th ? 1 : 2);
}

// The NPR consecutive pairs p0 .. p0+NPR-1 that one thread rotates, read from
// the rotary table of QkArgs::rope_tab (row stride 2*npairs floats: cos of
// every pair, then sin).  `axes` holds each pair's axis (2 bits per pair);
// `uni` says all of them share one axis, so their entries are adjacent in one
// table row and come in 16-byte loads.
template <int NPR>
struct TabPairs {
  int axes;
  bool uni;
  __device__ __forceinline__ void init(int p0, int sec_t, int sec_th) {
    axes = 0;
    const int a0 = pair_axis(p0, sec_t, sec_th);
    uni = true;
#pragma unroll
    for (int i = 0; i < NPR; ++i) {
      const int ax = pair_axis(p0 + i, sec_t, sec_th);
      axes |= ax << (2 * i);
      uni &= ax == a0;
    }
  }
  // c[i], s[i]: cos and sin of pair p0 + i at position (t, h, w)
  __device__ __forceinline__ void read(const float *tab, int npairs, int p0, int t, int h, int w,
                                       float (&c)[NPR], float (&s)[NPR]) const {
    const int64_t ld = 2 * static_cast<int64_t>(npairs);
    if (uni) {
      const int ax = axes & 3;
      const int at = ax == 0 ? t : (ax == 1 ? h : w);
      const float *row = tab + at * ld + p0;
      if constexpr (NPR % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NPR; i += 4) {
          const float4 cv = __ldg(reinterpret_cast<const float4 *>(row + i));
          const float4 sv = __ldg(reinterpret_cast<const float4 *>(row + npairs + i));
          c[i] = cv.x, c[i + 1] = cv.y, c[i + 2] = cv.z, c[i + 3] = cv.w;
          s[i] = sv.x, s[i + 1] = sv.y, s[i + 2] = sv.z, s[i + 3] = sv.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < NPR; i += 2) {
          const float2 cv = __ldg(reinterpret_cast<const float2 *>(row + i));
          const float2 sv = __ldg(reinterpret_cast<const float2 *>(row + npairs + i));
          c[i] = cv.x, c[i + 1] = cv.y;
          s[i] = sv.x, s[i + 1] = sv.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < NPR; ++i) {
        const int ax = (axes >> (2 * i)) & 3;
        const int at = ax == 0 ? t : (ax == 1 ? h : w);
        const float *row = tab + at * ld + p0 + i;
        c[i] = __ldg(row);
        s[i] = __ldg(row + npairs);
      }
    }
  }
};

// On-the-fly form: the (cos, sin) of the rotary angles of R consecutive rows,
// the first at the cursors (rows past the CTA's share are computed but never
// read), into cos_out/sin_out[R][kMaxPairs].  The angle pos * freq is formed
// and reduced modulo 2*pi in fp64, then sincosf runs on the reduced fp32
// angle.  The CTA's NT threads share the R * npairs entries.
template <int R, int NT>
__device__ __forceinline__ void angle_tables(const QkArgs &a, const double *freq, TokenCursor tok,
                                             GridCursor pos, float *cos_out, float *sin_out) {
  int pt[R], ph[R], pw[R];
#pragma unroll
  for (int q = 0; q < R; ++q) {
    pt[q] = pos.t;
    ph[q] = pos.h;
    pw[q] = pos.w;
    tok.next(a.L);
    pos.next(tok.r, a.n_video, a.H, a.W);
  }
  for (int idx = threadIdx.x; idx < R * a.npairs; idx += NT) {
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
    cos_out[q * kMaxPairs + p] = cv;
    sin_out[q * kMaxPairs + p] = sv;
  }
}

// Table form staged through shared memory (STAGE): the (cos, sin) of one
// row, copied from the rotary table into dst[2][kMaxPairs] with cp.async in
// the same group as the row's q and k, so their latency hides behind the
// ring's prefetch like the data's.  Threads c < npairs/4 copy the cos of
// pairs 4c .. 4c+3 (16 bytes when the four share an axis, else four 4-byte
// copies), threads npairs/4 + c their sin.  The row's position comes from
// its global index by division: the issuing threads run ahead of the
// consumer's row cursor.  Readers need a CTA barrier after the wait.
__device__ __forceinline__ void stage_table_row(const QkArgs &a, int64_t row, float *dst) {
  const int nq = a.npairs >> 2;
  if (static_cast<int>(threadIdx.x) >= 2 * nq) return;
  const int b = static_cast<int>(row / a.L);
  const int r = static_cast<int>(row - static_cast<int64_t>(b) * a.L);
  int t, h = 0, w = 0;
  if (r < a.n_video) {
    t = r / a.HW;
    const int rem = r - t * a.HW;
    h = rem / a.W;
    w = rem - h * a.W;
  } else {
    t = r - a.n_video;
  }
  const int64_t ld = 2 * static_cast<int64_t>(a.npairs);
  for (int idx = threadIdx.x; idx < 2 * nq; idx += blockDim.x) {
    const int which = idx >= nq ? 1 : 0;  // 0: cos, 1: sin
    const int p = 4 * (idx - which * nq);
    const float *src = a.rope_tab + which * a.npairs + p;
    float *d = dst + which * kMaxPairs + p;
    const int ax0 = pair_axis(p, a.sec_t, a.sec_th);
    if (ax0 == pair_axis(p + 3, a.sec_t, a.sec_th)) {
      const int at = ax0 == 0 ? t : (ax0 == 1 ? h : w);
      cp_async16_ca(d, src + at * ld);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int ax = pair_axis(p + i, a.sec_t, a.sec_th);
        const int at = ax == 0 ? t : (ax == 1 ? h : w);
        cp_async4(d + i, src + at * ld + i);
      }
    }
  }
}

// Bytes of shared memory before the ring: the fp64 frequency table and the
// per-row angle tables of the on-the-fly form, or STAGE's table ring of
// (S + 1) stages (one deeper than the data ring, so that a stage is only
// overwritten once every thread has passed the barrier after its last use).
template <int R, int S, bool TAB, bool STAGE>
__host__ __device__ constexpr size_t head_bytes() {
  return !TAB ? header_bytes<R>()
              : (STAGE ? static_cast<size_t>(S + 1) * R * 2 * kMaxPairs * 4 : 0);
}

template <typename T, int G, int NT, int VPT, int R, int S, bool TAB, int K = 0, bool BAR = false,
          bool STAGE = false>
__global__ void __launch_bounds__(NT) qknorm_rope3d_kernel(const QkArgs a) {
  static_assert(K % R == 0, "a ring stage's rows must lie in one chunk");
  using IO = Io<T>;
  constexpr int E = IO::E;
  constexpr int PPV = E / 2;  // rotary pairs per 16-byte vector
  constexpr int Q = PPV / 2;  // float2 lanes of (pair 2m, pair 2m+1) per vector
  // STAGE (table form only): each row's table entries ride in the ring
  // (stage_table_row) instead of each thread loading its own pairs per row
  constexpr bool DIRECT = TAB && !STAGE;
  constexpr int TS = S + 1;  // STAGE's table ring
  constexpr int NTAB = 2 * R * kMaxPairs;
  constexpr size_t HDR = head_bytes<R, S, TAB, STAGE>();
  extern __shared__ __align__(16) unsigned char smem[];
  double *freq = reinterpret_cast<double *>(smem);
  float *tabr = reinterpret_cast<float *>(smem);                  // STAGE: [TS][R][2][kMaxPairs]
  float *cosb = reinterpret_cast<float *>(smem + kMaxPairs * 8);  // [2][R][kMaxPairs]
  float *sinb = cosb + NTAB;                                      // [2][R][kMaxPairs]
  uint4 *ring = reinterpret_cast<uint4 *>(smem + HDR);            // [S][R][2][VPT][NT]

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
  TabPairs<PPV> tp;
  if constexpr (DIRECT) {
    tp.init(p0, a.sec_t, a.sec_th);
  } else if constexpr (!TAB) {
    for (int p = tid; p < a.npairs; p += NT)
      freq[p] = pow(static_cast<double>(a.theta), -2.0 * p / a.head_dim);
  }

  // chunks of at least 4 rows: each chunk restarts the row and position
  // cursors with divisions, which 1- or 2-row chunks made visible
  RowOrder<K, (K < 4 ? (K > R ? K : R) : 4)> ro;
  ro.init(a.rows);
  const int count = ro.count;
  const int iters = (count + R - 1) / R;
  auto slot = [&](int s, int q, int part, int k) -> uint4 * {
    return &ring[(((s * R + q) * 2 + part) * VPT + k) * NT + tid];
  };
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const unsigned char *src = qkv + ro.row(j) * a.ld_qkv_bytes;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint4 *ps = reinterpret_cast<const uint4 *>(src + part * part_bytes) + tid;
#pragma unroll
          for (int k = 0; k < VPT; ++k)
            if (ok[k]) cp_async16(slot(s, q, part, k), ps + k * NT);
        }
        if constexpr (STAGE)
          stage_table_row(a, ro.row(j), tabr + ((it % TS) * R + q) * 2 * kMaxPairs);
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < S - 1; ++s) issue(s, s);
  if constexpr (!TAB) __syncthreads();  // freq[] visible

  TokenCursor tok;
  GridCursor pos;
  int cons = 0;
  int buf = 0;
  for (int it = 0; it < iters; ++it) {
    issue(it + S - 1, cons == 0 ? S - 1 : cons - 1);
    if (ro.run_start(it * R)) {  // this stage's rows start a new run
      tok.init(ro.row(it * R), a.L);
      pos.init(tok.r, a.n_video, a.HW, a.W);
    }

    if constexpr (!TAB)
      angle_tables<R, NT>(a, freq, tok, pos, cosb + buf * R * kMaxPairs,
                          sinb + buf * R * kMaxPairs);

    cp_async_wait<S - 1>();
    if constexpr (!DIRECT || BAR) __syncthreads();  // angle tables of these rows visible

#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        // cs[m] = (cos of pair p0+2m, cos of pair p0+2m+1); likewise sn
        float2 cs[Q], sn[Q];
        if constexpr (DIRECT) {
          float c[PPV], s[PPV];
          tp.read(a.rope_tab, a.npairs, p0, pos.t, pos.h, pos.w, c, s);
#pragma unroll
          for (int m = 0; m < Q; ++m) {
            cs[m] = make_float2(c[2 * m], c[2 * m + 1]);
            sn[m] = make_float2(s[2 * m], s[2 * m + 1]);
          }
        } else if constexpr (STAGE) {
          const float *tr = tabr + ((it % TS) * R + q) * 2 * kMaxPairs + p0;
#pragma unroll
          for (int m = 0; m < Q; ++m) {
            cs[m] = *reinterpret_cast<const float2 *>(tr + 2 * m);
            sn[m] = *reinterpret_cast<const float2 *>(tr + kMaxPairs + 2 * m);
          }
        } else {
#pragma unroll
          for (int m = 0; m < Q; ++m) {
            cs[m] =
                *reinterpret_cast<const float2 *>(&cosb[(buf * R + q) * kMaxPairs + p0 + 2 * m]);
            sn[m] =
                *reinterpret_cast<const float2 *>(&sinb[(buf * R + q) * kMaxPairs + p0 + 2 * m]);
          }
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
              reinterpret_cast<uint4 *>((part == 0 ? qo : ko) + ro.row(j) * a.ld_out_bytes) + tid;
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

// One launch of a fixed configuration: a wave of as many CTAs as fit.
template <typename T, int G, int NT, int VPT, int R, int S, bool TAB, int K = 0, bool BAR = false,
          bool STAGE = false>
cudaError_t launch_cfg(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  const void *fn = reinterpret_cast<const void *>(
      &qknorm_rope3d_kernel<T, G, NT, VPT, R, S, TAB, K, BAR, STAGE>);
  const size_t smem =
      head_bytes<R, S, TAB, STAGE>() + static_cast<size_t>(S) * R * 2 * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  qknorm_rope3d_kernel<T, G, NT, VPT, R, S, TAB, K, BAR, STAGE>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

// Row order and ring of the two forms, measured at the 5 s clip on a B200
// at 1,965 MHz, 20-step runs after idling:
//  - Rows go to the CTAs in chunks dealt round-robin, so the whole grid
//    works through one contiguous window of the tensors; a contiguous share
//    per CTA (296 far-apart streams) ran in a slower DRAM mode, 0.91-0.92 ms
//    against 0.79-0.83 ms.
//  - On the fly: two rows per stage, two stages (the angle tables already
//    put one CTA barrier on every stage), chunks of 8 rows.
//  - Table-driven: one row per stage, three stages, chunks of 4 rows, and a
//    CTA barrier per stage although nothing is shared: it keeps the CTA's
//    warps on the same row, so each row is requested as one burst (0.84
//    against 0.90 ms without it at 256 x 3; 0.80 ms at 320 x 2).
constexpr int kOtfChunk = 8;
constexpr int kTabRows = 1;
constexpr int kTabStages = 3;
constexpr int kTabChunk = 4;

template <typename T, int G, int NT, int VPT>
cudaError_t launch(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  constexpr int R = VPT <= 6 ? 2 : 1;  // keeps the ring within shared memory
  return launch_cfg<T, G, NT, VPT, R, 2, false, kOtfChunk, false>(a, stream, geo);
}

template <typename T, int G>
cudaError_t dispatch(const QkArgs &a, int threads, int vpt, cudaStream_t stream, Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch<T, G, NT, V>(a, stream, geo);
  SOL_QK_OTF_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

template <typename T, int G>
cudaError_t dispatch_tab(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                         Geometry *geo) {
#define SOL_CASE(NT, V)          \
  if (threads == NT && vpt == V) \
    return launch_cfg<T, G, NT, V, kTabRows, kTabStages, true, kTabChunk, true>(a, stream, geo);
  SOL_QK_TAB_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

// Launch for element type T: the table-driven form (TAB, a.rope_tab set) or
// the on-the-fly one, G = head_dim * esize / 16 lanes per head.
template <typename T, bool TAB>
cudaError_t launch_form(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  const int G = a.head_dim * static_cast<int>(sizeof(T)) / 16;
  if (a.npairs > kMaxPairs || TAB != (a.rope_tab != nullptr)) return cudaErrorInvalidValue;
  int threads = 0, vpt = 0;
  if (!(TAB ? pick_split_tab : pick_split_otf)(a.nvec_q, &threads, &vpt))
    return cudaErrorInvalidValue;
  switch (G) {
#define SOL_G(g)                                                                  \
  case g:                                                                         \
    if constexpr (TAB) return dispatch_tab<T, g>(a, threads, vpt, stream, geo); \
    else return dispatch<T, g>(a, threads, vpt, stream, geo);
    SOL_G(2) SOL_G(4) SOL_G(8) SOL_G(16) SOL_G(32)
#undef SOL_G
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qk
}  // namespace sol
