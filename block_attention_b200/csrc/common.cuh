// common.cuh -- small device helpers shared by the Orthrus sm_100a kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "orthrus.h"

namespace orthrus {

// Record the first device-side error in the caller's optional error word.
__device__ __forceinline__ void set_err(int32_t* err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Four consecutive elements as float4; p must be aligned to 4 elements.
__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  float4 r;
  r.x = __uint_as_float(u.x << 16);
  r.y = __uint_as_float(u.x & 0xffff0000u);
  r.z = __uint_as_float(u.y << 16);
  r.w = __uint_as_float(u.y & 0xffff0000u);
  return r;
}

__host__ __device__ constexpr int ceil_div(int a, int b) { return (a + b - 1) / b; }

// RoPE (rotary position embedding) pieces shared by the stand-alone RoPE
// kernel and the QKV projection's epilogue, so that both give identical
// bits: the angle pos * theta^(-2i/hd) with its cosine and sine in double,
// rounded to float; the rotation of the pair (x1, x2) = (x[i], x[i + hd/2])
// in float with every rounding explicit (no contraction left to the
// compiler):  x1' = x1 c - x2 s,  x2' = x2 c + x1 s.
__device__ __forceinline__ float2 rope_cos_sin(int64_t pos, int i, int hd, double theta) {
  const double ang = (double)pos * pow(theta, -2.0 * i / hd);
  double sn, cn;
  sincos(ang, &sn, &cn);
  return make_float2((float)cn, (float)sn);
}
__device__ __forceinline__ float rope_first(float x1, float x2, float2 cs) {
  return __fmaf_rn(x1, cs.x, -__fmul_rn(x2, cs.y));
}
__device__ __forceinline__ float rope_second(float x1, float x2, float2 cs) {
  return __fmaf_rn(x2, cs.x, __fmul_rn(x1, cs.y));
}

}  // namespace orthrus
