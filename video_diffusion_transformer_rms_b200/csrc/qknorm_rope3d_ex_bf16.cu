// QKNorm + 3D RoPE epilogue variants with bf16 output, for head_dim 64, 128
// or 256 and either rotary pair layout.
#include "qknorm_rope3d_ex.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_ex_bf16out(const QkArgs &a, bool half_split, cudaStream_t stream,
                                           Geometry *geo) {
  return qk::launch_ex_form<false, false>(a, half_split, stream, geo);
}

}  // namespace sol
