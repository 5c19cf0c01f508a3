// common.cuh -- device helpers shared by the ReplaySSM kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/replayssm.h"

namespace rssm {

// Most records a buffer slot array may hold: window (<= 16) plus up to three
// extra slots for the tail of a speculative round (draft_max <= 4).
constexpr int kMaxCap = 20;
constexpr int kThreads = 256;  // 8 warps per CTA for every kernel here

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// First error wins: a zero status word takes the code, a non-zero one keeps
// the code it already holds.
__device__ __forceinline__ void report(int32_t *status, int32_t code) {
  if (status) atomicCAS(status, 0, code);
}

// 128-bit global loads/stores of fp32 state tiles.  The checkpoint is read
// once per step and is far larger than L2, so loads stream past L1 and stores
// are marked evict-first.
__device__ __forceinline__ float4 ld_stream(const float *p) {
  float4 v;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_stream(float *p, float4 v) {
  asm volatile("st.global.L1::no_allocate.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x),
               "f"(v.y), "f"(v.z), "f"(v.w)
               : "memory");
}

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

// v <- a * v and v <- x * b + v on a float4 as two paired fp32 operations
// (Blackwell's f32x2 pipe: per component the same rounding as fmulf / fmaf).
__device__ __forceinline__ float4 mul4x(float a, float4 v) {
  const float2 a2 = make_float2(a, a);
  const float2 lo = __fmul2_rn(a2, make_float2(v.x, v.y));
  const float2 hi = __fmul2_rn(a2, make_float2(v.z, v.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}
__device__ __forceinline__ float4 fma4x(float x, float4 b, float4 v) {
  const float2 x2 = make_float2(x, x);
  const float2 lo = __ffma2_rn(x2, make_float2(b.x, b.y), make_float2(v.x, v.y));
  const float2 hi = __ffma2_rn(x2, make_float2(b.z, b.w), make_float2(v.z, v.w));
  return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// Load element i of a step input stored as T.
template <typename T>
__device__ __forceinline__ float ld_in(const void *base, int64_t i) {
  return to_f32(static_cast<const T *>(base)[i]);
}

}  // namespace rssm
