// QKNorm + 3D RoPE reading (cos, sin) from a rotary table, instantiated for
// float I/O.
#include "qknorm_rope3d.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_tab_f32(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  return qk::launch_form<float, true>(a, stream, geo);
}

}  // namespace sol
