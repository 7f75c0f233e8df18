// Device-side helpers shared by the libsol kernels (sm_100a).
//
// Every kernel streams token rows HBM -> shared memory with cp.async
// (16-byte LDGSTS, L2-only, no register staging) in an S-stage ring per CTA,
// computes in fp32 registers and writes results back with 16-byte
// streaming stores.  Each thread copies and later consumes exactly the same
// 16-byte slots of every stage, so the ring needs no CTA barrier: a thread's
// own cp.async.wait_group is enough.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sol {

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy, cached in L2 only.
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// Wait until at most N of this thread's committed groups are still pending.
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// 16-byte store marked streaming (evict-first): results are not re-read here.
__device__ __forceinline__ void st_stream16(void *gmem_dst, const uint4 &v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"l"(gmem_dst), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Small vectors (modulation, gamma) that every CTA re-reads: read-only path,
// cached in L1.
__device__ __forceinline__ uint4 ld_shared_vec(const void *gmem_src) {
  return __ldg(reinterpret_cast<const uint4 *>(gmem_src));
}

// Element type traits: E elements per 16-byte vector, exact widening to fp32
// and round-to-nearest-even narrowing.
template <typename T>
struct Io;

template <>
struct Io<float> {
  static constexpr int E = 4;
  __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[E]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[E]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

template <>
struct Io<__nv_bfloat16> {
  static constexpr int E = 8;
  // bf16 is the upper half of a binary32 pattern: widening is a shift.
  __device__ __forceinline__ static void unpack2(uint32_t w, float &lo, float &hi) {
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xffff0000u);
  }
  __device__ __forceinline__ static uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low half) = lo
    return *reinterpret_cast<uint32_t *>(&h);
  }
  __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[E]) {
    unpack2(v.x, f[0], f[1]);
    unpack2(v.y, f[2], f[3]);
    unpack2(v.z, f[4], f[5]);
    unpack2(v.w, f[6], f[7]);
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[E]) {
    return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                      pack2(f[6], f[7]));
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over aligned groups of G lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace sol
