// QKNorm + 3D RoPE kernels instantiated for float I/O.
#include "qknorm_rope3d.cuh"

namespace sol {

cudaError_t launch_qknorm_rope3d_f32(const QkArgs &a, cudaStream_t stream, Geometry *geo) {
  using T = float;
  const int esize = sizeof(T);
  const int G = a.head_dim * esize / 16;  // lanes per head
  if (a.npairs > qk::kMaxPairs) return cudaErrorInvalidValue;
  int threads = 0, vpt = 0;
  if (!pick_split_qk(a.nvec_q, &threads, &vpt)) return cudaErrorInvalidValue;
  switch (G) {
    case 2: return qk::dispatch<T, 2>(a, threads, vpt, stream, geo);
    case 4: return qk::dispatch<T, 4>(a, threads, vpt, stream, geo);
    case 8: return qk::dispatch<T, 8>(a, threads, vpt, stream, geo);
    case 16: return qk::dispatch<T, 16>(a, threads, vpt, stream, geo);
    case 32: return qk::dispatch<T, 32>(a, threads, vpt, stream, geo);
    default: return cudaErrorInvalidValue;
  }
}


}  // namespace sol
