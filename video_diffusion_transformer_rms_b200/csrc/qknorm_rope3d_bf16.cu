// QKNorm + 3D RoPE, on-the-fly (cos, sin), instantiated for __nv_bfloat16 I/O.
#include "qknorm_rope3d.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_bf16(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  return qk::launch_form<__nv_bfloat16, false>(a, stream, geo);
}

}  // namespace sol
