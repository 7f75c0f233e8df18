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
  // Interleaved INT8 reduces its sum of squares and max side by side, one
  // shuffle chain per vector, so it takes the row-reduction split (up to 6
  // vectors per thread: 128 x 5 at D = 5120, which divides the row exactly)
  // rather than the QK rule's 256 x 3, which leaves a sixth of the vector
  // slots empty; measured 0.86 against 0.97 ms inside a step.  The
  // half-split variant keeps the QK rule.
  const bool split = half_split ? pick_split_qk(a.nvec_q, &threads, &vpt)
                                : pick_split(a.nvec_q, &threads, &vpt);
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
