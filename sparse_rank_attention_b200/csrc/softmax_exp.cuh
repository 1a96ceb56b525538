// Exponentials and packing of the attention kernels' softmax (head dim 128, sm_100a):
// P = 2^x with x = s * scale * log2(e) - m <= 0, written as fp16 pairs or e4m3 quads.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace rola {

// 2^x on the special-function unit (ex2.approx: relative error ~2^-22, 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA and integer pipes, leaving the special-function unit to the other
// exponentials: x = n + f with n = round(x) (1.5 * 2^23 added and taken away), f in
// [-0.5, 0.5]; 2^f from a cubic least-squares fit at Chebyshev nodes (relative error
// below 7.8e-5, under half an fp16 ulp); 2^n added into the exponent field.  x is clamped
// to -125 (results below 2^-125 are not needed: P is e4m3 where this is used), so -inf
// gives 2^-125 rather than 0; the callers use it for scores that are finite.
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;
  const float n = t - 12582912.f;
  const float fr = x - n;
  const float p = fmaf(fmaf(fmaf(0.05508868f, fr, 0.24260405f), fr, 0.69327623f), fr, 0.99992895f);
  // t's low mantissa bits hold n; shifting by 23 drops the rest of t's bits
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Four floats to four e4m3 bytes (round to nearest even, saturating to +-448).
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

}  // namespace rola
