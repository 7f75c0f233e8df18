// Device-side helpers shared by the libsol kernels (sm_100a).
//
// Every kernel streams token rows HBM -> shared memory with cp.async
// (16-byte LDGSTS, L2-only, no register staging) in an S-stage ring per CTA,
// computes in fp32 registers with Blackwell's packed fp32x2 FMA/MUL (two
// lanes of arithmetic per instruction) and writes results back with 16-byte
// streaming stores.  Each thread copies and later consumes exactly the same
// 16-byte slots of every stage, so the ring needs no CTA barrier: a thread's
// own cp.async.wait_group is enough.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sol {

// ---------------------------------------------------------------------------
// memory movement
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy, cached in L2 only.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

// 4-byte global -> shared copy through L1 (the .cg form copies 16 bytes only).
__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

// 16-byte global -> shared copy through L1 (for small data many CTAs re-read).
__device__ __forceinline__ void cp_async16_ca(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// Wait until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// 16-byte store marked streaming (evict-first): results are not re-read here.
__device__ __forceinline__ void st_stream16(void *gmem_dst, const uint4 &v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"l"(gmem_dst), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Small vectors (modulation, gamma) that every CTA re-reads: read-only path,
// cached in L1.
__device__ __forceinline__ uint4 ld_shared_vec(const void *gmem_src) {
  return __ldg(reinterpret_cast<const uint4 *>(gmem_src));
}

// ---------------------------------------------------------------------------
// packed fp32x2 arithmetic (one instruction for two lanes on sm_100)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// ---------------------------------------------------------------------------
// element types: a 16-byte vector holds E elements = E/2 natural pairs
// (elements 2i, 2i+1).  Widening is exact, narrowing rounds to nearest even.
// ---------------------------------------------------------------------------

template <typename T>
struct Io;

template <>
struct Io<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void unpack(const uint4 &v, float2 (&p)[2]) {
    p[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
    p[1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
  }
  __device__ __forceinline__ static uint4 pack(const float2 (&p)[2]) {
    return make_uint4(__float_as_uint(p[0].x), __float_as_uint(p[0].y), __float_as_uint(p[1].x),
                      __float_as_uint(p[1].y));
  }
  // Rotary split: ev[m] = (x[4m], x[4m+2]), od[m] = (x[4m+1], x[4m+3]), so
  // that lane 0 / lane 1 of each float2 belong to rotary pairs 2m / 2m+1.
  __device__ __forceinline__ static void unpack_eo(const uint4 &v, float2 (&ev)[1],
                                                   float2 (&od)[1]) {
    ev[0] = make_float2(__uint_as_float(v.x), __uint_as_float(v.z));
    od[0] = make_float2(__uint_as_float(v.y), __uint_as_float(v.w));
  }
  // Inverse of unpack_eo for the rotated pair components u0 (first) / u1.
  __device__ __forceinline__ static uint4 pack_eo(const float2 (&u0)[1], const float2 (&u1)[1]) {
    return make_uint4(__float_as_uint(u0[0].x), __float_as_uint(u1[0].x),
                      __float_as_uint(u0[0].y), __float_as_uint(u1[0].y));
  }
};

template <>
struct Io<__nv_bfloat16> {
  static constexpr int E = 8;
  // bf16 is the upper half of a binary32 pattern: widening is a shift / mask.
  __device__ __forceinline__ static float lo(uint32_t w) { return __uint_as_float(w << 16); }
  __device__ __forceinline__ static float hi(uint32_t w) {
    return __uint_as_float(w & 0xffff0000u);
  }
  __device__ __forceinline__ static uint32_t pack2(float l, float h) {
    __nv_bfloat162 b = __floats2bfloat162_rn(l, h);  // .x (low half) = l
    return *reinterpret_cast<uint32_t *>(&b);
  }
  __device__ __forceinline__ static void unpack(const uint4 &v, float2 (&p)[4]) {
    p[0] = make_float2(lo(v.x), hi(v.x));
    p[1] = make_float2(lo(v.y), hi(v.y));
    p[2] = make_float2(lo(v.z), hi(v.z));
    p[3] = make_float2(lo(v.w), hi(v.w));
  }
  __device__ __forceinline__ static uint4 pack(const float2 (&p)[4]) {
    return make_uint4(pack2(p[0].x, p[0].y), pack2(p[1].x, p[1].y), pack2(p[2].x, p[2].y),
                      pack2(p[3].x, p[3].y));
  }
  __device__ __forceinline__ static void unpack_eo(const uint4 &v, float2 (&ev)[2],
                                                   float2 (&od)[2]) {
    ev[0] = make_float2(lo(v.x), lo(v.y));
    od[0] = make_float2(hi(v.x), hi(v.y));
    ev[1] = make_float2(lo(v.z), lo(v.w));
    od[1] = make_float2(hi(v.z), hi(v.w));
  }
  __device__ __forceinline__ static uint4 pack_eo(const float2 (&u0)[2], const float2 (&u1)[2]) {
    return make_uint4(pack2(u0[0].x, u1[0].x), pack2(u0[0].y, u1[0].y), pack2(u0[1].x, u1[1].x),
                      pack2(u0[1].y, u1[1].y));
  }
};

// ---------------------------------------------------------------------------
// reductions
// ---------------------------------------------------------------------------

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over aligned groups of G lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// row bookkeeping
// ---------------------------------------------------------------------------

// Contiguous share [begin, begin + count) of `rows` for CTA `cta` out of
// `ctas`; the shares differ by at most one row.  A share is walked with a
// 32-bit local row index (the host rejects sizes that would overflow it).
__device__ __forceinline__ void cta_rows(int64_t rows, int64_t cta, int64_t ctas,
                                         int64_t &begin, int &count) {
  begin = rows * cta / ctas;
  count = static_cast<int>(rows * (cta + 1) / ctas - begin);
}

// The rows one CTA streams, in order.  K == 0: the CTA's contiguous share
// (cta_rows).  K > 0: chunks of consecutive rows dealt round-robin, chunk c
// to CTA c mod gridDim.x, so that at any moment the grid works through one
// contiguous window of the tensors instead of gridDim.x far-apart streams.
// The chunk is K rows, halved (down to KMIN, at least the rows of one ring
// stage) while the CTAs would get fewer than 16 chunks each: with few rows
// per CTA a large chunk leaves some CTAs one chunk more than others, a tail
// of up to K rows.  K and KMIN are powers of two.  Rows within a chunk (or a
// share) are consecutive.
template <int K, int KMIN = 1>
struct RowOrder {
  static_assert(K == 0 || (K % KMIN == 0 && (K & (K - 1)) == 0 && (KMIN & (KMIN - 1)) == 0),
                "chunk sizes are powers of two");
  int64_t begin;  // K == 0: first row of the share
  int count;      // rows of this CTA
  int ks;         // log2 of the chunk size
  int cta, ctas;  // this CTA's index among the CTAs that share the rows
  __device__ __forceinline__ void init(int64_t rows) { init(rows, blockIdx.x, gridDim.x); }
  __device__ __forceinline__ void init(int64_t rows, int cta_, int ctas_) {
    cta = cta_;
    ctas = ctas_;
    if constexpr (K == 0) {
      cta_rows(rows, cta, ctas, begin, count);
      ks = 0;
    } else {
      int k = K;
      while (k > KMIN && rows < static_cast<int64_t>(ctas) * k * 16) k >>= 1;
      ks = 31 - __clz(k);
      const int64_t chunks = (rows + k - 1) >> ks, c = cta, g = ctas;
      const int64_t mine = c < chunks ? (chunks - 1 - c) / g + 1 : 0;
      int64_t n = mine << ks;
      if (mine > 0 && c + (mine - 1) * g == chunks - 1) n -= (chunks << ks) - rows;  // last
      begin = 0;
      count = static_cast<int>(n);
    }
  }
  // global index of the CTA's j-th row
  __device__ __forceinline__ int64_t row(int j) const {
    if constexpr (K == 0) {
      return begin + j;
    } else {
      return ((static_cast<int64_t>(j >> ks) * ctas + cta) << ks) + (j & ((1 << ks) - 1));
    }
  }
  // row j is the first of a run of consecutive rows (row cursors restart)
  __device__ __forceinline__ bool run_start(int j) const {
    if constexpr (K == 0) {
      return j == 0;
    } else {
      return (j & ((1 << ks) - 1)) == 0;
    }
  }
};

// (sample b, row r in the sample) of a global row, advanced one row at a
// time: one division per CTA instead of one per row.  L < 2^31.
struct TokenCursor {
  int b, r;
  __device__ __forceinline__ void init(int64_t row, int L) {
    b = static_cast<int>(row / L);
    r = static_cast<int>(row - static_cast<int64_t>(b) * L);
  }
  __device__ __forceinline__ void next(int L) {
    if (++r == L) {
      r = 0;
      ++b;
    }
  }
};

// 3D rotary position (t, h, w) of the row a TokenCursor points at: video
// rows r < n_video walk the T x H x W grid in raster order (t-major), audio
// row i = r - n_video sits at (i, 0, 0).
struct GridCursor {
  int t, h, w;
  __device__ __forceinline__ void init(int r, int n_video, int HW, int W) {
    if (r < n_video) {
      t = r / HW;
      const int rem = r - t * HW;
      h = rem / W;
      w = rem - h * W;
    } else {
      t = r - n_video;
      h = 0;
      w = 0;
    }
  }
  // Move to row r_next (= r + 1, or 0 when a new sample starts).
  __device__ __forceinline__ void next(int r_next, int n_video, int H, int W) {
    if (r_next == 0 || r_next == n_video) {
      t = 0;
      h = 0;
      w = 0;
    } else if (r_next < n_video) {
      if (++w == W) {
        w = 0;
        if (++h == H) {
          h = 0;
          ++t;
        }
      }
    } else {
      ++t;
    }
  }
};

// ---- INT8 codes ---------------------------------------------------------

// Round-half-even of x*s for |x*s| <= 127 by adding 1.5 * 2^23: the fp32
// sum has an ulp of 1, so one FMA rounds the exact product to an integer and
// leaves it, as a two's-complement byte, in the low byte of the bit pattern.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

// Low bytes of four words, in order, as one word.
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// 8-byte streaming store (evict-first, like st_stream16).
__device__ __forceinline__ void st_stream8(void *gmem_dst, uint32_t lo, uint32_t hi) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};\n" ::"l"(gmem_dst), "r"(lo), "r"(hi)
               : "memory");
}

}  // namespace sol
