// QKNorm + 3D RoPE reading (cos, sin) from a rotary table, instantiated for
// __nv_bfloat16 I/O.
#include "qknorm_rope3d.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_tab_bf16(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  return qk::launch_form<__nv_bfloat16, true>(a, stream, geo);
}

}  // namespace sol
