// Per-head symmetric INT8 quantisation of bf16 head vectors: the v part of a
// merged QKV row for the INT8 Q/K/V exchange between GPUs that the KOCPC
// Sol-H3 article's 4x/8x B300 runs use.  For each token row and head h
// (channels [h*hd, (h+1)*hd) of the row):
//   scale = max|x| / 127,  code = round_half_even(x * 127 / max|x|)
// (scale 0 and all codes 0 for an all-zero head), codes in the same layouts as
// the QKNorm+RoPE epilogue's INT8 q and k.
//
// Memory-bound: 2 bytes read and 1 byte written per element.  Persistent
// CTAs walk the rows in round-robin chunks; a thread owns VPT 16-byte
// vectors of a row (G consecutive lanes per head) and keeps the next row's
// vectors in flight in registers while it quantises the current one.  The
// head's max is a G-lane shuffle max; the codes are rounded by one packed FMA
// with 1.5 * 2^23 and packed with byte permutes, as in the INT8 epilogue.
#include "sol_device.cuh"
#include "sol_launch.h"

namespace sol {
namespace {

template <int G, int NT, int VPT, int K = 0, bool FULL = false>
__global__ void __launch_bounds__(NT) quantize_heads_kernel(const QuantArgs a) {
  using IO = Io<__nv_bfloat16>;
  constexpr int E = IO::E;  // 8 elements per vector
  constexpr int P = E / 2;
  const int tid = threadIdx.x;
  const int gl = tid % G;

  // uniform over each head's G lanes (nvec and NT are multiples of G);
  // FULL: the split covers the row exactly, no access needs a guard
  bool ok[VPT];
  int64_t off[VPT];
#pragma unroll
  for (int k = 0; k < VPT; ++k) {
    const int v = k * NT + tid;
    ok[k] = FULL || v < a.nvec;
    off[k] = static_cast<int64_t>(v / G) * a.out_sh + (v % G) * 8;
  }

  RowOrder<K> ro;
  ro.init(a.rows);
  const int count = ro.count;
  if (count == 0) return;
  const unsigned char *src = static_cast<const unsigned char *>(a.src);
  auto load = [&](int j, uint4 (&x)[VPT]) {
    const uint4 *row = reinterpret_cast<const uint4 *>(src + ro.row(j) * a.ld_src_bytes) + tid;
#pragma unroll
    for (int k = 0; k < VPT; ++k) x[k] = ok[k] ? __ldcs(row + k * NT) : make_uint4(0, 0, 0, 0);
  };

  TokenCursor tok;
  uint4 cur[VPT], nxt[VPT];
  load(0, cur);
  for (int j = 0; j < count; ++j) {
    if (ro.run_start(j)) tok.init(ro.row(j), a.L);
    if (j + 1 < count) load(j + 1, nxt);
    unsigned char *orow = static_cast<unsigned char *>(a.out) +
                          static_cast<int64_t>(tok.b) * a.out_sb +
                          static_cast<int64_t>(tok.r) * a.out_sr;
    float *srow = a.scale + ro.row(j) * static_cast<int64_t>(a.n_heads);
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
      float2 x[P];
      IO::unpack(cur[k], x);
      float m4[P];
#pragma unroll
      for (int m = 0; m < P; ++m) m4[m] = fmaxf(fabsf(x[m].x), fabsf(x[m].y));
      float xmax = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
#pragma unroll
      for (int o = G / 2; o > 0; o >>= 1)
        xmax = fmaxf(xmax, __shfl_xor_sync(0xffffffffu, xmax, o));
      // |x * is| <= 127 up to the fast division's 2 ulp, which the
      // round-to-nearest keeps at 127
      float is = xmax > 0.f ? __fdividef(127.f, xmax) : 0.f;
      if (xmax > 0.f && xmax < 0x1p-96f) {
        // a head of (near-)denormal values: 127 / xmax would overflow, so
        // scale x and xmax by 2^64 (exact) first; the codes are unchanged
#pragma unroll
        for (int m = 0; m < P; ++m) x[m] = mul2(x[m], splat2(0x1p64f));
        is = __fdividef(127.f, xmax * 0x1p64f);
      }
      uint32_t c[E];
      const float2 is2 = splat2(is), magic2 = splat2(kRoundMagic);
#pragma unroll
      for (int m = 0; m < P; ++m) {
        const float2 r = fma2(x[m], is2, magic2);
        c[2 * m] = __float_as_uint(r.x);
        c[2 * m + 1] = __float_as_uint(r.y);
      }
      if (ok[k]) {
        st_stream8(orow + off[k], pack_low_bytes(c[0], c[1], c[2], c[3]),
                   pack_low_bytes(c[4], c[5], c[6], c[7]));
        if (gl == 0) srow[(k * NT + tid) / G] = xmax * (1.f / 127.f);
      }
    }
    tok.next(a.L);
#pragma unroll
    for (int k = 0; k < VPT; ++k) cur[k] = nxt[k];
  }
}

// Rows in chunks of 8 dealt round-robin over the CTAs (RowOrder), as the
// other streaming kernels: 0.348 against 0.362 ms for contiguous shares at
// the 5 s clip, codes and scales bit-identical.
template <int G, int NT, int VPT, bool FULL, int K = 8>
cudaError_t launch_t(const QuantArgs &a, cudaStream_t stream, Geometry *geo) {
  if (FULL && a.nvec != NT * VPT) return cudaErrorInvalidValue;
  const void *fn = reinterpret_cast<const void *>(&quantize_heads_kernel<G, NT, VPT, K, FULL>);
  const int per_sm = resident_blocks(fn, NT, 0);
  if (per_sm <= 0) return cudaErrorInvalidConfiguration;
  int64_t grid = static_cast<int64_t>(per_sm) * device_sms();
  if (grid > a.rows) grid = a.rows;
  if (geo) *geo = Geometry{NT, VPT, 1, 0, static_cast<int>(grid)};
  quantize_heads_kernel<G, NT, VPT, K, FULL><<<static_cast<unsigned>(grid), NT, 0, stream>>>(a);
  return cudaGetLastError();
}

// A split that covers the row exactly (128 x 5 at D = 5120) takes the
// unguarded instantiation (FULL): INT8 q, k and v at the 5 s clip 1.039 ->
// 1.008 ms in one interleaved session (the q/k kernel unchanged), codes
// bit-identical.
template <int G>
cudaError_t dispatch(const QuantArgs &a, int threads, int vpt, cudaStream_t stream,
                     Geometry *geo) {
#define SOL_CASE(NT, V)                                                \
  if (threads == NT && vpt == V)                                       \
    return a.nvec == NT * V ? launch_t<G, NT, V, true>(a, stream, geo) \
                            : launch_t<G, NT, V, false>(a, stream, geo);
  SOL_SPLITS(SOL_CASE)
#undef SOL_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_quantize_heads_int8(const QuantArgs &a, int head_dim, cudaStream_t stream,
                                       Geometry *geo) {
  int threads = 0, vpt = 0;
  if (!pick_split(a.nvec, &threads, &vpt)) return cudaErrorInvalidValue;
  switch (head_dim * 2 / 16) {
    case 8: return dispatch<8>(a, threads, vpt, stream, geo);
    case 16: return dispatch<16>(a, threads, vpt, stream, geo);
    case 32: return dispatch<32>(a, threads, vpt, stream, geo);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sol
