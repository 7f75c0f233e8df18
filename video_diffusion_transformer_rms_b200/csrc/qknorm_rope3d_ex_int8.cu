// QKNorm + 3D RoPE epilogue variants with INT8 (+ fp32 scale) output, for
// head_dim 64, 128 or 256 (G = 8, 16, 32 lanes per head) and either rotary
// pair layout.
#include "qknorm_rope3d_ex.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_ex_int8out(const QkArgs &a, bool half_split, cudaStream_t stream,
                                           Geometry *geo) {
  const int G = a.head_dim * 2 / 16;
  if (a.npairs > qk::kMaxPairs) return cudaErrorInvalidValue;
  int threads = 0, vpt = 0;
  // the split rule of qk::kRowSplit, which dispatch_ex instantiates
  const bool row = half_split ? qk::kRowSplit<true, true> : qk::kRowSplit<false, true>;
  const bool split = row ? pick_split(a.nvec_q, &threads, &vpt)
                         : pick_split_qk(a.nvec_q, &threads, &vpt);
  if (!split) return cudaErrorInvalidValue;
  switch (G) {
    case 8:
      return half_split ? qk::dispatch_ex<8, true, true>(a, threads, vpt, stream, geo)
                        : qk::dispatch_ex<8, false, true>(a, threads, vpt, stream, geo);
    case 16:
      return half_split ? qk::dispatch_ex<16, true, true>(a, threads, vpt, stream, geo)
                        : qk::dispatch_ex<16, false, true>(a, threads, vpt, stream, geo);
    case 32:
      return half_split ? qk::dispatch_ex<32, true, true>(a, threads, vpt, stream, geo)
                        : qk::dispatch_ex<32, false, true>(a, threads, vpt, stream, geo);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace sol
