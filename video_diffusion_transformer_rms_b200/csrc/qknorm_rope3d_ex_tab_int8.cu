// QKNorm + 3D RoPE epilogue variants with INT8 (+ fp32 scale) output and
// (cos, sin) read from a rotary table, for head_dim 64, 128 or 256 and
// either pair layout.
#include "qknorm_rope3d_ex.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_ex_tab_int8out(const QkArgs &a, bool half_split,
                                               cudaStream_t stream, Geometry *geo) {
  return qk::launch_ex_form<true, true>(a, half_split, stream, geo);
}

}  // namespace sol
