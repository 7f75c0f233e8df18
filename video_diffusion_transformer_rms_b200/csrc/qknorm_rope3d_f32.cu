// QKNorm + 3D RoPE, on-the-fly (cos, sin), instantiated for float I/O.
#include "qknorm_rope3d.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_f32(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  return qk::launch_form<float, false>(a, stream, geo);
}

}  // namespace sol
