// lsa_common.cuh -- helpers shared by the sm_100a kernels of the LSA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/lsa.h"

namespace lsa {

// First nonzero status written wins; later ones are dropped.
__device__ __forceinline__ void set_status(int32_t* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements starting at p (p 8-byte aligned for bf16, 16-byte
// aligned for fp32) as floats.
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  float4 t = __ldg(reinterpret_cast<const float4*>(p));
  v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
  uint2 t = __ldg(reinterpret_cast<const uint2*>(p));
  __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&t.x);
  __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&t.y);
  float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
  v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}
__device__ __forceinline__ void load2(const float* p, float (&v)[2]) {
  float2 t = __ldg(reinterpret_cast<const float2*>(p));
  v[0] = t.x; v[1] = t.y;
}
__device__ __forceinline__ void load2(const __nv_bfloat16* p, float (&v)[2]) {
  __nv_bfloat162 t = __ldg(reinterpret_cast<const __nv_bfloat162*>(p));
  float2 f = __bfloat1622float2(t);
  v[0] = f.x; v[1] = f.y;
}

// Two consecutive elements through a generic pointer (global or shared memory).
__device__ __forceinline__ void load2_generic(const float* p, float (&v)[2]) {
  const float2 t = *reinterpret_cast<const float2*>(p);
  v[0] = t.x; v[1] = t.y;
}
__device__ __forceinline__ void load2_generic(const __nv_bfloat16* p, float (&v)[2]) {
  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
  v[0] = f.x; v[1] = f.y;
}

// Order-preserving map of a float to uint32 (larger float -> larger uint);
// -0.0 is folded onto +0.0 so the two never order differently.
__device__ __forceinline__ uint32_t orderable(float f) {
  if (f == 0.0f) f = 0.0f;
  uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): output i (0-based) of the
// generator whose state starts at s is mix(s + (i + 1) * gamma).
__host__ __device__ __forceinline__ uint64_t splitmix64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}
__host__ __device__ __forceinline__ uint64_t splitmix64_at(uint64_t s, uint64_t i) {
  return splitmix64_mix(s + (i + 1) * 0x9e3779b97f4a7c15ULL);
}

__host__ __device__ __forceinline__ int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

}  // namespace lsa
