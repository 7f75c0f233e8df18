// QKNorm + 3D RoPE epilogue variants (bf16 input), for what consumes q and k
// next:
//   - any output layout with unit element stride: per (sample, token row,
//     head) strides, e.g. attention's [B, H, L, head_dim] straight away;
//   - the half-split rotary pair layout, pair i = elements (i, i + hd/2);
//   - INT8 output: symmetric per-(row, head) codes round(x * 127 / max|x|)
//     with fp32 scales max|x| / 127, the quantised Q/K that the KOCPC Sol-H3
//     article's 4x/8x B300 runs send between GPUs;
//   - a per-axis frequency ladder: each of the t/h/w sections a RoPE of its
//     own, pair j of a section of s pairs at theta^(-j/s).
// Same structure as qknorm_rope3d.cuh (ring, cursors, per-row angle tables or
// the precomputed rotary table (TAB), G lanes per head).  With the half-split layout a thread's partner elements
// (i + hd/2, or i - hd/2) sit in lane gl ^ G/2 of the same head: one 16-byte
// shuffle per vector brings them over, and each thread writes only its own
// elements.  With INT8 output the head's max |x| is a G-lane shuffle max,
// run side by side with the sum of squares (the 1/rms factor cancels from
// the codes); the codes are rounded half to even from the fp32 value (one FMA
// with a magic constant, then byte permutes).
#pragma once
#include "qknorm_rope3d.cuh"

namespace sol {
namespace qk {

// INT8 codes of one lane's 2 * NV rotated values of a head, held as NV
// float2 in the registers the rotation leaves them in, whose other values
// sit in the G - 1 partner lanes of its aligned lane group.  ROT: v[2w] and
// v[2w + 1] are the first and the second components of two rotary pairs
// (elements 4w, 4w+2 and 4w+1, 4w+3), as the interleaved rotation produces
// them; else v[i] holds elements 2i, 2i+1.  Taking them as they are keeps the
// packed rounding FMAs free of register moves.  1/rms is one positive factor
// per head, so it cancels from the codes: code = round(u * 127 / max|u|) on
// the un-normalised rotation, and only the scale max|u| / rms / 127 needs it.
// The sum of squares (ssq: this lane's part) and the max reduce side by side.
// Codes are rounded half to even (one FMA with kRoundMagic) and packed four
// to a word, in element order.
template <int NV, int G, bool ROT>
__device__ __forceinline__ void int8_codes(float2 (&v)[NV], float ssq, float inv_hd, float eps,
                                           uint32_t (&words)[NV / 2], float &scale) {
  constexpr int W = NV / 2;  // words, 4 elements each
  float m[W];
#pragma unroll
  for (int w = 0; w < W; ++w)
    m[w] = fmaxf(fmaxf(fabsf(v[2 * w].x), fabsf(v[2 * w].y)),
                 fmaxf(fabsf(v[2 * w + 1].x), fabsf(v[2 * w + 1].y)));
#pragma unroll
  for (int k = W / 2; k > 0; k >>= 1)
#pragma unroll
    for (int e = 0; e < k; ++e) m[e] = fmaxf(m[e], m[e + k]);
  float umax = m[0];
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) {
    ssq += __shfl_xor_sync(0xffffffffu, ssq, off);
    umax = fmaxf(umax, __shfl_xor_sync(0xffffffffu, umax, off));
  }
  const float inv = rsqrtf(fmaf(ssq, inv_hd, eps));
  // |u * is| <= 127 up to the fast division's 2 ulp, which the round to
  // nearest keeps at 127
  float is = umax > 0.f ? __fdividef(127.f, umax) : 0.f;
  if (umax > 0.f && umax < 0x1p-96f) {
    // a head of (near-)denormal inputs: 127 / umax would overflow, so scale
    // u and umax by 2^64 (exact) first; the codes are unchanged
    const float2 big = splat2(0x1p64f);
#pragma unroll
    for (int e = 0; e < NV; ++e) v[e] = mul2(v[e], big);
    is = __fdividef(127.f, umax * 0x1p64f);
  }
  const float2 is2 = splat2(is), magic2 = splat2(kRoundMagic);
#pragma unroll
  for (int w = 0; w < W; ++w) {
    const float2 r0 = fma2(v[2 * w], is2, magic2);
    const float2 r1 = fma2(v[2 * w + 1], is2, magic2);
    words[w] = ROT ? pack_low_bytes(__float_as_uint(r0.x), __float_as_uint(r1.x),
                                    __float_as_uint(r0.y), __float_as_uint(r1.y))
                   : pack_low_bytes(__float_as_uint(r0.x), __float_as_uint(r0.y),
                                    __float_as_uint(r1.x), __float_as_uint(r1.y));
  }
  scale = umax * inv * (1.f / 127.f);
}

template <int G, int NT, int VPT, int R, int S, bool HALF, bool OUT8, bool TAB, int K = 0,
          bool BAR = false, bool STAGE = false, bool FULL = false>
__global__ void __launch_bounds__(NT) qknorm_rope3d_ex_kernel(const QkArgs a) {
  static_assert(K % R == 0, "a ring stage's rows must lie in one chunk");
  using IO = Io<__nv_bfloat16>;
  constexpr int E = IO::E;    // 8 elements per 16-byte vector
  constexpr int P = E / 2;    // natural pairs (2e, 2e+1)
  constexpr int Q = P / 2;    // float2 lanes of two rotary pairs (interleaved layout)
  constexpr int VB = OUT8 ? 8 : 16;  // output bytes per vector
  constexpr int NPR = HALF ? E : P;  // rotary pairs of one thread's vector
  // STAGE (table form only): each row's table entries ride in the ring
  // (stage_table_row) instead of each thread loading its own pairs per row
  constexpr bool DIRECT = TAB && !STAGE;
  constexpr int TS = S + 1;  // STAGE's table ring
  constexpr int NTAB = 2 * R * kMaxPairs;
  constexpr size_t HDR = head_bytes<R, S, TAB, STAGE>();
  extern __shared__ __align__(16) unsigned char smem[];
  double *freq = reinterpret_cast<double *>(smem);
  float *tabr = reinterpret_cast<float *>(smem);  // STAGE: [TS][R][2][kMaxPairs]
  float *cosb = reinterpret_cast<float *>(smem + kMaxPairs * 8);
  float *sinb = cosb + NTAB;
  uint4 *ring = reinterpret_cast<uint4 *>(smem + HDR);

  const int tid = threadIdx.x;
  const int gl = tid % G;
  // first rotary pair of this thread's elements: interleaved, E/2 pairs per
  // vector; half-split, one pair per element, positions mod hd/2
  const int p0 = HALF ? (gl % (G / 2)) * E : gl * (E / 2);
  const int64_t part_bytes = static_cast<int64_t>(a.nvec_q) * 16;

  // FULL: the split covers a part's vectors exactly (NT * VPT == nvec_q),
  // so no access needs a guard
  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = FULL || k * NT + tid < a.nvec_q;

  // gamma: interleaved as in qknorm_rope3d.cuh; half-split as own / partner
  // elements in natural pairs
  float2 gev[2][Q], god[2][Q];   // interleaved
  float2 gown[2][P], gpar[2][P]; // half-split
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const uint4 *g = static_cast<const uint4 *>(part == 0 ? a.gamma_q : a.gamma_k);
    if constexpr (HALF) {
      if (g) {
        IO::unpack(ld_shared_vec(g + gl), gown[part]);
        IO::unpack(ld_shared_vec(g + (gl ^ (G / 2))), gpar[part]);
      } else {
#pragma unroll
        for (int m = 0; m < P; ++m) gown[part][m] = gpar[part][m] = splat2(1.f);
      }
    } else {
      if (g) {
        IO::unpack_eo(ld_shared_vec(g + gl), gev[part], god[part]);
      } else {
#pragma unroll
        for (int m = 0; m < Q; ++m) gev[part][m] = god[part][m] = splat2(1.f);
      }
    }
  }
  // frequency of each rotary pair: one ladder over all pairs, or with
  // per_axis one per section (local pair j of a section of s pairs at
  // theta^(-j/s))
  TabPairs<NPR> tp;
  if constexpr (DIRECT) {
    tp.init(p0, a.sec_t, a.sec_th);
  } else if constexpr (!TAB) {
    for (int p = tid; p < a.npairs; p += NT) {
      double e = -2.0 * p / a.head_dim;
      if (a.per_axis) {
        const int start = p < a.sec_t ? 0 : (p < a.sec_th ? a.sec_t : a.sec_th);
        const int size = p < a.sec_t ? a.sec_t : (p < a.sec_th ? a.sec_th - a.sec_t
                                                               : a.npairs - a.sec_th);
        e = -static_cast<double>(p - start) / size;
      }
      freq[p] = pow(static_cast<double>(a.theta), e);
    }
  }

  // chunks of at least 4 rows: each chunk restarts the row and position
  // cursors with divisions, which 1- or 2-row chunks made visible
  RowOrder<K, (K < 4 ? (K > R ? K : R) : 4)> ro;
  ro.init(a.rows);
  const int count = ro.count;
  const int iters = (count + R - 1) / R;
  const unsigned char *qkv = static_cast<const unsigned char *>(a.qkv);
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
  if constexpr (!TAB) __syncthreads();

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
    if constexpr (!DIRECT || BAR) __syncthreads();

#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        // cos and sin of this thread's NPR pairs p0 .. p0 + NPR - 1
        float ct[NPR], st[NPR];
        if constexpr (DIRECT) {
          tp.read(a.rope_tab, a.npairs, p0, pos.t, pos.h, pos.w, ct, st);
        } else if constexpr (STAGE) {
          const float *tr = tabr + ((it % TS) * R + q) * 2 * kMaxPairs + p0;
#pragma unroll
          for (int i = 0; i < NPR; ++i) {
            ct[i] = tr[i];
            st[i] = tr[kMaxPairs + i];
          }
        } else {
#pragma unroll
          for (int i = 0; i < NPR; ++i) {
            ct[i] = cosb[(buf * R + q) * kMaxPairs + p0 + i];
            st[i] = sinb[(buf * R + q) * kMaxPairs + p0 + i];
          }
        }
        const int64_t row_off = static_cast<int64_t>(tok.b) * a.out_sb +
                                static_cast<int64_t>(tok.r) * a.out_sr;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          // rotation coefficients of this thread's elements, gamma folded in
          float2 c0[Q], ns1[Q], s0[Q], c1[Q];  // interleaved
          float2 ca[P], sb[P];                 // half-split: own*c + partner*(+-s)
          if constexpr (HALF) {
            const float sgn = gl >= G / 2 ? 1.f : -1.f;
#pragma unroll
            for (int m = 0; m < P; ++m) {
              const float2 cc = make_float2(ct[2 * m], ct[2 * m + 1]);
              const float2 ss = make_float2(st[2 * m], st[2 * m + 1]);
              ca[m] = mul2(gown[part][m], cc);
              sb[m] = mul2(gpar[part][m], make_float2(sgn * ss.x, sgn * ss.y));
            }
          } else {
#pragma unroll
            for (int m = 0; m < Q; ++m) {
              const float2 cs = make_float2(ct[2 * m], ct[2 * m + 1]);
              const float2 sn = make_float2(st[2 * m], st[2 * m + 1]);
              c0[m] = mul2(gev[part][m], cs);
              s0[m] = mul2(gev[part][m], sn);
              ns1[m] = mul2(god[part][m], make_float2(-sn.x, -sn.y));
              c1[m] = mul2(god[part][m], cs);
            }
          }
          unsigned char *obase = static_cast<unsigned char *>(part == 0 ? a.q_out : a.k_out) +
                                 row_off;
          float *scale_row = OUT8 ? (part == 0 ? a.q_scale : a.k_scale) +
                                        ro.row(j) * static_cast<int64_t>(a.n_heads)
                                  : nullptr;
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            const int v = k * NT + tid;
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (ok[k]) xv = *slot(cons, q, part, k);
            // rotated outputs, not yet multiplied by the head's 1/rms, as the
            // rotation leaves them in registers: half-split, uv[m] = elements
            // (2m, 2m+1); interleaved, uv[2m] / uv[2m+1] = first / second
            // components of pairs 2m and 2m+1.  acc: this thread's part of
            // the sum of squares
            float2 uv[P];
            float2 acc;
            if constexpr (HALF) {
              uint4 pv;
              pv.x = __shfl_xor_sync(0xffffffffu, xv.x, G / 2);
              pv.y = __shfl_xor_sync(0xffffffffu, xv.y, G / 2);
              pv.z = __shfl_xor_sync(0xffffffffu, xv.z, G / 2);
              pv.w = __shfl_xor_sync(0xffffffffu, xv.w, G / 2);
              float2 own[P], par[P];
              IO::unpack(xv, own);
              IO::unpack(pv, par);
              acc = mul2(own[0], own[0]);
#pragma unroll
              for (int m = 1; m < P; ++m) acc = fma2(own[m], own[m], acc);
#pragma unroll
              for (int m = 0; m < P; ++m) {
                uv[m] = fma2(own[m], ca[m], mul2(par[m], sb[m]));
              }
            } else {
              float2 ev[Q], od[Q];
              IO::unpack_eo(xv, ev, od);
              acc = mul2(ev[0], ev[0]);
              acc = fma2(od[0], od[0], acc);
#pragma unroll
              for (int m = 1; m < Q; ++m) {
                acc = fma2(ev[m], ev[m], acc);
                acc = fma2(od[m], od[m], acc);
              }
#pragma unroll
              for (int m = 0; m < Q; ++m) {
                uv[2 * m] = fma2(od[m], ns1[m], mul2(ev[m], c0[m]));
                uv[2 * m + 1] = fma2(od[m], c1[m], mul2(ev[m], s0[m]));
              }
            }
            const int head = v / G;
            unsigned char *dst = obase + static_cast<int64_t>(head) * a.out_sh + (v % G) * VB;
            if constexpr (OUT8) {
              uint32_t w8[2];
              float scale;
              int8_codes<P, G, !HALF>(uv, acc.x + acc.y, a.inv_hd, a.eps, w8, scale);
              if (ok[k]) {
                st_stream8(dst, w8[0], w8[1]);
                if (gl == 0) scale_row[head] = scale;
              }
            } else {
              const float2 inv2 = splat2(rsqrtf(fmaf(group_sum<G>(acc.x + acc.y), a.inv_hd, a.eps)));
              float2 pr[P];
#pragma unroll
              for (int m = 0; m < P; ++m) pr[m] = mul2(uv[m], inv2);
              // a plain (evict-normal) store: in head-strided layouts such as
              // [B, H, L, hd] consecutive rows of a head are adjacent, and L2
              // can merge a CTA's successive rows before writing back (4%
              // faster there than evict-first; the same in [B, L, H, hd])
              if (ok[k]) {
                if constexpr (HALF) {
                  *reinterpret_cast<uint4 *>(dst) = IO::pack(pr);
                } else {
                  const float2 f0[Q] = {pr[0], pr[2]}, f1[Q] = {pr[1], pr[3]};
                  *reinterpret_cast<uint4 *>(dst) = IO::pack_eo(f0, f1);
                }
              }
            }
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

// The CTA split each variant of qknorm_rope3d_ex_kernel takes, measured
// inside a step at the 5 s clip: the row-reduction rule (pick_split, <= 6
// vectors per thread: 128 x 5 at D = 5120, which divides the row exactly)
// for half-split bf16 from the table (0.92 against 0.97 ms; on the fly it
// takes dispatch_ex_half_otf); the QK rule (pick_split_qk:
// 256 x 3, more warps, a sixth of the vector slots empty) for interleaved
// bf16 and half-split INT8.  (Interleaved INT8 runs in
// qknorm_rope3d_int8w_kernel, split by pick_split_i8w.)
template <bool HALF, bool OUT8>
constexpr bool kRowSplit = HALF != OUT8;

// Table form of qknorm_rope3d_int8w_kernel: the warp's lanes copy the (cos,
// sin) of one row at rotary position (t, h, w) into the warp's own
// dst[2][kMaxPairs], one 16-byte chunk per lane and round (chunk c <
// npairs/4: cos of pairs 4c .. 4c+3, then the sin chunks), in the cp.async
// group of the row's data.  Only this warp reads them, so a __syncwarp after
// the wait orders them and the CTA needs no barrier per stage.
__device__ __forceinline__ void stage_table_lanes(const QkArgs &a, int t, int h, int w,
                                                  float *dst, int lane) {
  const int nq = a.npairs >> 2;
  const int64_t ld = 2 * static_cast<int64_t>(a.npairs);
  for (int idx = lane; idx < 2 * nq; idx += 32) {
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

// Shared memory before qknorm_rope3d_int8w_kernel's ring: the table form's
// per-warp table rows, (S + 1) stages deep (a stage is overwritten only after
// every lane of the warp passed the __syncwarp that follows its last use), or
// the on-the-fly form's fp64 frequencies and double-buffered angle tables.
template <int R, int S, bool TAB, int NT>
__host__ __device__ constexpr size_t i8w_head_bytes() {
  return TAB ? static_cast<size_t>(S + 1) * (NT / 32) * R * 2 * kMaxPairs * 4 : header_bytes<R>();
}

// INT8 output with interleaved pairs, 16 elements per lane.  The INT8
// epilogue is bound by instruction issue and latency, not DRAM, and most of
// its per-element cost is per head and lane: the two-value shuffle
// reduction, the reciprocals and the scale store.  Here G2 = head_dim / 16
// lanes share a head (8 at head_dim 128), and lane g owns the head's 16-byte
// chunks g and g + G2, i.e. pairs 4g .. 4g+3 and 4(g+G2) .. 4(g+G2)+3.  A
// warp's copy of the first chunks covers whole 128-byte halves of four heads,
// so every L2 sector it touches is used in full, and the second copy the
// other halves.  The reduction runs over G2 lanes for 16 elements instead of
// 2 * G2 lanes for 8.  Codes go out as two 8-byte stores per lane.
//
// PSPLIT: CTA 2i takes the q part and CTA 2i + 1 the k part of the same rows
// (one row order for the pair), so a CTA holds half a row per ring stage and
// one part's gamma.  The table form stages each row's (cos, sin) per warp
// (stage_table_lanes) and has no CTA barrier in its loop; the on-the-fly form
// builds CTA-wide angle tables behind one barrier per stage.
template <int G2, int NT, int VPT, int R, int S, bool TAB, int K = 0, int MINB = 1,
          bool PSPLIT = true, bool FULL = false>
__global__ void __launch_bounds__(NT, MINB) qknorm_rope3d_int8w_kernel(const QkArgs a) {
  static_assert(K % R == 0, "a ring stage's rows must lie in one chunk");
  static_assert(NT % 32 == 0 && 32 % G2 == 0, "a head's lanes must share a warp");
  using IO = Io<__nv_bfloat16>;
  constexpr int P = 4;       // rotary pairs per 16-byte chunk
  constexpr int Q = 2;       // float2 lanes of (pair 2m, pair 2m+1) per chunk
  constexpr int TS = S + 1;  // the table form's ring of per-warp table rows
  constexpr int NW = NT / 32;
  constexpr int NTAB = 2 * R * kMaxPairs;
  constexpr size_t HDR = i8w_head_bytes<R, S, TAB, NT>();
  extern __shared__ __align__(16) unsigned char smem[];
  double *freq = reinterpret_cast<double *>(smem);                // on the fly
  float *cosb = reinterpret_cast<float *>(smem + kMaxPairs * 8);  // on the fly: [2][R][kMaxPairs]
  float *sinb = cosb + NTAB;
  float *tabw = reinterpret_cast<float *>(smem);  // table: [TS][NW][R][2][kMaxPairs]
  constexpr int NP = PSPLIT ? 1 : 2;
  const int pbase = PSPLIT ? static_cast<int>(blockIdx.x & 1) : 0;
  uint4 *ring = reinterpret_cast<uint4 *>(smem + HDR);  // [S][R][NP][VPT][2][NT]

  const int tid = threadIdx.x;
  const int g = tid % G2;
  const int warp = tid >> 5, lane = tid & 31;
  const int nslots = a.nvec_q / 2;  // (head, lane) slots of one part: n_heads * G2
  const int64_t part_bytes = static_cast<int64_t>(a.nvec_q) * 16;
  int p0[2];  // first pair of each half
  p0[0] = P * g;
  p0[1] = P * (g + G2);

  // FULL: the split covers a part's slots exactly (NT * VPT == nslots), so
  // every slot is real and no access needs a guard
  bool ok[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) ok[k] = FULL || k * NT + tid < nslots;
  // output address of slot k: the slot-0 head of this lane plus k * hstep
  const int64_t hstep = static_cast<int64_t>(NT / G2) * a.out_sh;

  // gamma per part and half in rotary layout, as qknorm_rope3d.cuh
  float2 gev[NP][2][Q], god[NP][2][Q];
#pragma unroll
  for (int pi = 0; pi < NP; ++pi) {
    const int part = pbase + pi;
    const uint4 *gp = static_cast<const uint4 *>(part == 0 ? a.gamma_q : a.gamma_k);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      if (gp) {
        IO::unpack_eo(ld_shared_vec(gp + g + h * G2), gev[pi][h], god[pi][h]);
      } else {
#pragma unroll
        for (int m = 0; m < Q; ++m) gev[pi][h][m] = god[pi][h][m] = splat2(1.f);
      }
    }
  }
  if constexpr (!TAB) {
    for (int p = tid; p < a.npairs; p += NT) {
      double e = -2.0 * p / a.head_dim;
      if (a.per_axis) {
        const int start = p < a.sec_t ? 0 : (p < a.sec_th ? a.sec_t : a.sec_th);
        const int size = p < a.sec_t ? a.sec_t : (p < a.sec_th ? a.sec_th - a.sec_t
                                                               : a.npairs - a.sec_th);
        e = -static_cast<double>(p - start) / size;
      }
      freq[p] = pow(static_cast<double>(a.theta), e);
    }
  }

  // chunks of at least 4 rows: each chunk restarts the row and position
  // cursors with divisions, which 1- or 2-row chunks made visible
  RowOrder<K, (K < 4 ? (K > R ? K : R) : 4)> ro;
  if constexpr (PSPLIT) {
    ro.init(a.rows, static_cast<int>(blockIdx.x >> 1), static_cast<int>(gridDim.x >> 1));
  } else {
    ro.init(a.rows);
  }
  const int count = ro.count;
  const int iters = (count + R - 1) / R;
  const unsigned char *qkv = static_cast<const unsigned char *>(a.qkv);
  auto slot = [&](int s, int q, int pi, int k, int h) -> uint4 * {
    return &ring[((((s * R + q) * NP + pi) * VPT + k) * 2 + h) * NT + tid];
  };
  // chunk index in a part of the first chunk of slot k: head * 2 * G2 + g
  auto chunk0 = [&](int k) -> int {
    const int u = k * NT + tid;
    return (u / G2) * (2 * G2) + g;
  };
  // the table form's table row of issue iteration it, row q, for this warp
  auto wtab = [&](int it, int q) -> float * {
    return tabw + (((it % TS) * NW + warp) * R + q) * 2 * kMaxPairs;
  };
  TokenCursor itok;  // table form: the row being issued, S - 1 rows ahead
  GridCursor ipos;
  auto issue = [&](int it, int s) {
#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        const unsigned char *src = qkv + ro.row(j) * a.ld_qkv_bytes;
#pragma unroll
        for (int pi = 0; pi < NP; ++pi) {
          const uint4 *ps = reinterpret_cast<const uint4 *>(src + (pbase + pi) * part_bytes);
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            if (ok[k]) {
              const int c = chunk0(k);
              cp_async16(slot(s, q, pi, k, 0), ps + c);
              cp_async16(slot(s, q, pi, k, 1), ps + c + G2);
            }
          }
        }
        if constexpr (TAB) {
          if (ro.run_start(j)) {
            itok.init(ro.row(j), a.L);
            ipos.init(itok.r, a.n_video, a.HW, a.W);
          }
          stage_table_lanes(a, ipos.t, ipos.h, ipos.w, wtab(it, q), lane);
          itok.next(a.L);
          ipos.next(itok.r, a.n_video, a.H, a.W);
        }
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
    if (ro.run_start(it * R)) {
      tok.init(ro.row(it * R), a.L);
      if constexpr (!TAB) pos.init(tok.r, a.n_video, a.HW, a.W);
    }
    if constexpr (!TAB)
      angle_tables<R, NT>(a, freq, tok, pos, cosb + buf * R * kMaxPairs,
                          sinb + buf * R * kMaxPairs);
    cp_async_wait<S - 1>();
    if constexpr (TAB) {
      __syncwarp();  // the warp's table row visible to all its lanes
    } else {
      __syncthreads();  // angle tables of these rows visible
    }

#pragma unroll
    for (int q = 0; q < R; ++q) {
      const int j = it * R + q;
      if (j < count) {
        // cos and sin of the lane's pairs, per half (16-byte aligned: p0 is
        // a multiple of 4 pairs and table rows are kMaxPairs long)
        float ct[2][P], st[2][P];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float *cr = TAB ? wtab(it, q) + p0[h] : cosb + (buf * R + q) * kMaxPairs + p0[h];
          const float *sr = TAB ? cr + kMaxPairs : sinb + (buf * R + q) * kMaxPairs + p0[h];
          const float4 c4 = *reinterpret_cast<const float4 *>(cr);
          const float4 s4 = *reinterpret_cast<const float4 *>(sr);
          ct[h][0] = c4.x, ct[h][1] = c4.y, ct[h][2] = c4.z, ct[h][3] = c4.w;
          st[h][0] = s4.x, st[h][1] = s4.y, st[h][2] = s4.z, st[h][3] = s4.w;
        }
        const int64_t grow = ro.row(j);
        const int64_t row_off = static_cast<int64_t>(tok.b) * a.out_sb +
                                static_cast<int64_t>(tok.r) * a.out_sr;
#pragma unroll
        for (int pi = 0; pi < NP; ++pi) {
          const int part = pbase + pi;
          // rotation coefficients of this lane's pairs, gamma folded in
          float2 c0[2][Q], ns1[2][Q], s0[2][Q], c1[2][Q];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int m = 0; m < Q; ++m) {
              const float2 cs = make_float2(ct[h][2 * m], ct[h][2 * m + 1]);
              const float2 sn = make_float2(st[h][2 * m], st[h][2 * m + 1]);
              c0[h][m] = mul2(gev[pi][h][m], cs);
              s0[h][m] = mul2(gev[pi][h][m], sn);
              ns1[h][m] = mul2(god[pi][h][m], make_float2(-sn.x, -sn.y));
              c1[h][m] = mul2(god[pi][h][m], cs);
            }
          }
          unsigned char *obase = static_cast<unsigned char *>(part == 0 ? a.q_out : a.k_out) +
                                 row_off + static_cast<int64_t>(tid / G2) * a.out_sh;
          float *scale_row = (part == 0 ? a.q_scale : a.k_scale) +
                             grow * static_cast<int64_t>(a.n_heads);
#pragma unroll
          for (int k = 0; k < VPT; ++k) {
            // every lane joins the shuffles; ok[] only guards memory accesses
            float2 uv[8];  // rotation pairs as produced: (u0, u1) of chunk h, pairs 2m, 2m+1
            float2 acc = splat2(0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint4 xv = make_uint4(0u, 0u, 0u, 0u);
              if (ok[k]) xv = *slot(cons, q, pi, k, h);
              float2 ev[Q], od[Q];
              IO::unpack_eo(xv, ev, od);
#pragma unroll
              for (int m = 0; m < Q; ++m) {
                acc = fma2(ev[m], ev[m], acc);
                acc = fma2(od[m], od[m], acc);
              }
#pragma unroll
              for (int m = 0; m < Q; ++m) {
                const float2 u0 = fma2(od[m], ns1[h][m], mul2(ev[m], c0[h][m]));
                const float2 u1 = fma2(od[m], c1[h][m], mul2(ev[m], s0[h][m]));
                uv[4 * h + 2 * m] = u0;
                uv[4 * h + 2 * m + 1] = u1;
              }
            }
            uint32_t w8[4];
            float scale;
            int8_codes<8, G2, true>(uv, acc.x + acc.y, a.inv_hd, a.eps, w8, scale);
            if (ok[k]) {
              const int head = (k * NT + tid) / G2;
              unsigned char *dst = obase + k * hstep;
              st_stream8(dst + g * 8, w8[0], w8[1]);
              st_stream8(dst + (g + G2) * 8, w8[2], w8[3]);
              if (g == 0) scale_row[head] = scale;
            }
          }
        }
        tok.next(a.L);
        if constexpr (!TAB) pos.next(tok.r, a.n_video, a.H, a.W);
      }
    }
    buf ^= 1;
    cons = (cons + 1 == S) ? 0 : cons + 1;
  }
  cp_async_wait<0>();
}

template <int G2, int NT, int VPT, int R, int S, bool TAB, int K = 0, int MINB = 1,
          bool PSPLIT = true, bool FULL = false>
cudaError_t launch_int8w_cfg(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  if (FULL && a.nvec_q / 2 != NT * VPT) return cudaErrorInvalidValue;
  const void *fn = reinterpret_cast<const void *>(
      &qknorm_rope3d_int8w_kernel<G2, NT, VPT, R, S, TAB, K, MINB, PSPLIT, FULL>);
  constexpr int NP = PSPLIT ? 1 : 2;
  const size_t smem =
      i8w_head_bytes<R, S, TAB, NT>() + static_cast<size_t>(S) * R * NP * VPT * 2 * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (PSPLIT) {  // pairs of CTAs (q, k) over the same rows
    grid &= ~static_cast<int64_t>(1);
    if (grid > 2 * a.rows) grid = 2 * a.rows;
    if (grid < 2) grid = 2;
  } else if (grid > a.rows) {
    grid = a.rows;
  }
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  qknorm_rope3d_int8w_kernel<G2, NT, VPT, R, S, TAB, K, MINB, PSPLIT, FULL>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

// One launch of a fixed configuration: a wave of as many CTAs as fit.
template <int G, int NT, int VPT, int R, int S, bool HALF, bool OUT8, bool TAB, int K = 0,
          bool BAR = false, bool STAGE = false, bool FULL = false>
cudaError_t launch_ex_cfg(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  if (FULL && a.nvec_q != NT * VPT) return cudaErrorInvalidValue;
  const void *fn = reinterpret_cast<const void *>(
      &qknorm_rope3d_ex_kernel<G, NT, VPT, R, S, HALF, OUT8, TAB, K, BAR, STAGE, FULL>);
  const size_t smem =
      head_bytes<R, S, TAB, STAGE>() + static_cast<size_t>(S) * R * 2 * VPT * NT * 16;
  const int per_sm = resident_blocks(fn, NT, smem);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, S, smem, static_cast<int>(grid)};
  qknorm_rope3d_ex_kernel<G, NT, VPT, R, S, HALF, OUT8, TAB, K, BAR, STAGE, FULL>
      <<<static_cast<unsigned>(grid), NT, smem, stream>>>(a);
  return cudaGetLastError();
}

// Ring and row order of the variants (standalone loops at the 5 s clip on a
// B200; the split is kRowSplit's for both forms):
//  - on the fly: one row per ring stage for INT8 and half-split bf16 (half
//    the ring, more CTAs per SM; INT8 0.90 against 1.04 ms), two for
//    interleaved bf16; rows in round-robin chunks of kExOtfChunk for bf16
//    output (32 rows: each CTA writes longer runs of a head's rows in
//    [B, H, L, hd], 0.922 -> 0.872 ms against chunks of 8, which had beaten
//    contiguous shares; half-split the same for 8 to 32), a contiguous share
//    per CTA for INT8, which is bound by instruction issue rather than DRAM
//    and gained nothing from chunks (0.84 against 0.80 ms);
//  - table-driven: one row per stage, two stages, chunks of kTabChunk and
//    a barrier per stage, each thread reading its table entries: 0.809 ms
//    half-split (6.4 TB/s).  (Interleaved bf16 from the table takes
//    dispatch_ex_tab_interleaved, interleaved INT8 dispatch_i8w.)
//  - a table-form split that covers a part's vectors exactly (FULL, 128 x 5
//    and 320 x 2 at D = 5120) drops the guards: half-split 0.863 -> 0.812
//    ms, [B, H, L, hd] 0.862 -> 0.836 ms in one session; the on-the-fly
//    half-split measured 2% slower unguarded and keeps its guards.
constexpr int kExOtfChunk = 32;

template <int G, int NT, int VPT, bool HALF, bool OUT8, bool TAB>
cudaError_t launch_ex(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  if constexpr (TAB) {
    // a split with no slot past the row's end takes the unguarded kernel
    return a.nvec_q == NT * VPT
               ? launch_ex_cfg<G, NT, VPT, 1, 2, HALF, OUT8, true, kTabChunk, true, false, true>(
                     a, stream, geo)
               : launch_ex_cfg<G, NT, VPT, 1, 2, HALF, OUT8, true, kTabChunk, true, false, false>(
                     a, stream, geo);
  } else {
    constexpr int R = (OUT8 || HALF) ? 1 : (VPT <= 6 ? 2 : 1);
    constexpr int K = OUT8 ? 0 : kExOtfChunk;
    return launch_ex_cfg<G, NT, VPT, R, 2, HALF, OUT8, false, K, false>(a, stream, geo);
  }
}

template <int G, bool HALF, bool OUT8, bool TAB>
cudaError_t dispatch_ex(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                        Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch_ex<G, NT, V, HALF, OUT8, TAB>(a, stream, geo);
  if constexpr (kRowSplit<HALF, OUT8>) {
    SOL_SPLITS(SOL_CASE)
  } else {
    SOL_QK_SPLITS(SOL_CASE)
  }
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

// Table form of interleaved bf16 output: the table's split (pick_split_tab,
// 320 x 2 at D = 5120), one row per stage, two stages, chunks of kTabChunk,
// table entries staged through the ring (STAGE): 0.844 ms in [B, H, L, hd]
// at the 5 s clip, against 0.885 ms for the QK split with direct table
// reads and 0.856 ms on the fly, in one session.
template <int G>
cudaError_t dispatch_ex_tab_interleaved(const QkArgs &a, int threads, int vpt,
                                        cudaStream_t stream, Geometry *geo) {
#define SOL_CASE(NT, V)                                                                       \
  if (threads == NT && vpt == V)                                                              \
    return a.nvec_q == NT * V                                                                 \
               ? launch_ex_cfg<G, NT, V, 1, 2, false, false, true, kTabChunk, true, true, true>( \
                     a, stream, geo)                                                          \
               : launch_ex_cfg<G, NT, V, 1, 2, false, false, true, kTabChunk, true, true,       \
                               false>(a, stream, geo);
  SOL_QK_TAB_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

// Half-split bf16 on the fly: the on-the-fly QK split (pick_split_otf, 160 x
// 4 at D = 5120, one row per stage): 0.906 -> 0.876 ms at the 5 s clip in
// one interleaved session against the row-reduction split (128 x 5); for
// [B, H, L, hd] interleaved output 160 x 4 was 8% slower than 256 x 3.
template <int G>
cudaError_t dispatch_ex_half_otf(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                                 Geometry *geo) {
#define SOL_CASE(NT, V) \
  if (threads == NT && vpt == V) return launch_ex<G, NT, V, true, false, false>(a, stream, geo);
  SOL_QK_OTF_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

// Interleaved INT8 with 16 elements per lane (qknorm_rope3d_int8w_kernel),
// G2 = head_dim / 16 lanes per head: one row per stage, two stages and a
// contiguous share of rows per CTA in both forms (chunks measured no gain),
// split by pick_split_i8w, q and k on paired CTAs (half the ring and gamma
// registers per CTA: table form 0.800 -> 0.739 ms, on the fly 0.699 ->
// 0.688 ms in one session).  Both forms cap registers at 128 (512 threads'
// worth of CTAs per SM: on the fly 0.707 -> 0.690 ms).  The table form
// stages each row's table entries per warp, which drops the CTA barrier from
// its loop: 0.781 -> 0.706 ms in one interleaved session at the 5 s clip
// (staging per CTA behind a barrier, or lanes reading the table themselves,
// were the slower alternatives).  A split that covers a part's slots
// exactly (64 x 5 at D = 5120) takes the unguarded instantiation (FULL):
// 0.708 -> 0.661 ms with the table, 0.704 -> 0.648 ms on the fly, in one
// session.
template <int G2, bool TAB>
cudaError_t dispatch_i8w(const QkArgs &a, int threads, int vpt, cudaStream_t stream,
                         Geometry *geo) {
#define SOL_CASE(NT, V)                                                                     \
  if (threads == NT && vpt == V)                                                            \
    return a.nvec_q / 2 == NT * V                                                           \
               ? launch_int8w_cfg<G2, NT, V, 1, 2, TAB, 0, 512 / NT, true, true>(a, stream, geo) \
               : launch_int8w_cfg<G2, NT, V, 1, 2, TAB, 0, 512 / NT, true, false>(a, stream, geo);
  SOL_I8W_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

// Launch of one output type (OUT8: int8 codes, else bf16) in one form (TAB:
// a.rope_tab set), for head_dim 64, 128 or 256 (G = 8, 16, 32 lanes per
// head) and either rotary pair layout.
template <bool OUT8, bool TAB>
cudaError_t launch_ex_form(const QkArgs &a, bool half, cudaStream_t stream, Geometry *geo) {
  const int G = a.head_dim * 2 / 16;
  if (a.npairs > kMaxPairs || TAB != (a.rope_tab != nullptr)) return cudaErrorInvalidValue;
  int threads = 0, vpt = 0;
  if constexpr (OUT8) {
    if (!half) {  // interleaved INT8: 16 elements per lane, G / 2 lanes per head
      if (!pick_split_i8w(a.nvec_q / 2, &threads, &vpt)) return cudaErrorInvalidValue;
      switch (G) {
        case 8: return dispatch_i8w<4, TAB>(a, threads, vpt, stream, geo);
        case 16: return dispatch_i8w<8, TAB>(a, threads, vpt, stream, geo);
        case 32: return dispatch_i8w<16, TAB>(a, threads, vpt, stream, geo);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  if constexpr (TAB && !OUT8) {
    if (!half) {  // interleaved bf16 from the table: its own split, staged entries
      if (!pick_split_tab(a.nvec_q, &threads, &vpt)) return cudaErrorInvalidValue;
      switch (G) {
        case 8: return dispatch_ex_tab_interleaved<8>(a, threads, vpt, stream, geo);
        case 16: return dispatch_ex_tab_interleaved<16>(a, threads, vpt, stream, geo);
        case 32: return dispatch_ex_tab_interleaved<32>(a, threads, vpt, stream, geo);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  if constexpr (!TAB && !OUT8) {
    if (half) {  // half-split bf16 on the fly: the on-the-fly QK split
      if (!pick_split_otf(a.nvec_q, &threads, &vpt)) return cudaErrorInvalidValue;
      switch (G) {
        case 8: return dispatch_ex_half_otf<8>(a, threads, vpt, stream, geo);
        case 16: return dispatch_ex_half_otf<16>(a, threads, vpt, stream, geo);
        case 32: return dispatch_ex_half_otf<32>(a, threads, vpt, stream, geo);
        default: return cudaErrorInvalidValue;
      }
    }
  }
  // the split rule of kRowSplit, which dispatch_ex instantiates
  const bool row = half ? kRowSplit<true, OUT8> : kRowSplit<false, OUT8>;
  const bool split =
      row ? pick_split(a.nvec_q, &threads, &vpt) : pick_split_qk(a.nvec_q, &threads, &vpt);
  if (!split) return cudaErrorInvalidValue;
  switch (G) {
#define SOL_G(g)                                                                     \
  case g:                                                                            \
    if constexpr (OUT8 || TAB) { /* interleaved: returned above */                    \
      return dispatch_ex<g, true, OUT8, TAB>(a, threads, vpt, stream, geo);          \
    } else {                                                                         \
      return half ? dispatch_ex<g, true, OUT8, TAB>(a, threads, vpt, stream, geo)    \
                  : dispatch_ex<g, false, OUT8, TAB>(a, threads, vpt, stream, geo);  \
    }
    SOL_G(8) SOL_G(16) SOL_G(32)
#undef SOL_G
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace qk
}  // namespace sol
