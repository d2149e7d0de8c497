// Shared device/host helpers of the MoE layer kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// ----------------------------------------------------------------------------- element types
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte vector of N elements of T, unpacked to / packed from fp32.
template <typename T> struct Vec16 {
  static constexpr int N = 16 / sizeof(T);
  uint4 raw;
  __device__ __forceinline__ void to_float(float* f) const {
    const T* p = reinterpret_cast<const T*>(&raw);
#pragma unroll
    for (int i = 0; i < N; ++i) f[i] = Elem<T>::to_f(p[i]);
  }
  __device__ __forceinline__ void from_float(const float* f) {
    T* p = reinterpret_cast<T*>(&raw);
#pragma unroll
    for (int i = 0; i < N; ++i) p[i] = Elem<T>::from_f(f[i]);
  }
};

__device__ __forceinline__ uint4 ldg16(const void* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}
// streaming load (read once): do not keep in L1
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ void stg16(void* p, uint4 v) {
  *reinterpret_cast<uint4*>(p) = v;
}

__device__ __forceinline__ void set_status(int* status, int bits) {
  if (status) atomicOr(status, bits);
}

// Programmatic dependent launch.  A kernel started with launch_pdl may be scheduled
// while the kernel before it in the stream drains; pdl_wait(), before its first access
// to global memory, waits for that kernel's completion and the visibility of all its
// writes, so the data dependences are those of an ordinary launch.  pdl_trigger() lets
// the next such kernel be scheduled once every CTA of this one has called it or exited
// (placed at the end of the work: earlier, the next kernel's CTAs would take SM slots
// while this one still has CTAs to place).  Both do nothing in an ordinary launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// fp32 value rounded to the nearest TF32 value (10 explicit mantissa bits, ties away from
// zero; the low 13 bits come out zero).  GEMM operands of the fp32 dtype are rounded
// where they are produced, so the tensor core (which reads fp32 operands as TF32 by
// dropping those bits) sees values it represents exactly, instead of truncating them
// towards zero.
__device__ __forceinline__ float tf32_round(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}
// The same for the four floats of a 16-byte vector.
__device__ __forceinline__ uint4 tf32_round4(uint4 v) {
  return make_uint4(__float_as_uint(tf32_round(__uint_as_float(v.x))),
                    __float_as_uint(tf32_round(__uint_as_float(v.y))),
                    __float_as_uint(tf32_round(__uint_as_float(v.z))),
                    __float_as_uint(tf32_round(__uint_as_float(v.w))));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace moe
