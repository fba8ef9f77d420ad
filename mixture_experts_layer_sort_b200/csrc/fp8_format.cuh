// fp8_format.cuh - the two 8-bit floating-point code formats of the FP8 layers:
// E4M3 (4 exponent, 3 mantissa bits; largest finite 448) and E5M2 (5 exponent,
// 2 mantissa bits; largest finite 57344), "smaller range but higher precision"
// against "larger range but lower precision" (kongchang.com, "MoE Kernel
// Engineering Optimization Practices on Amazon SageMaker AI", section "Triton
// Backend Routing: A Practical Path to FP8 Quantization").
//
// Per-tensor scales: s = amax / (largest finite value), s = 1 for an all-zero
// tensor; codes = round-to-nearest-even(v / s) with the division in IEEE fp32,
// saturated to the largest finite value. The value of each format is also its
// operand-format code in a tcgen05 kind::f8f6f4 instruction descriptor.
#pragma once

#include <cuda_fp8.h>

namespace moe {

enum Fp8Format : int { kFp8E4M3 = 0, kFp8E5M2 = 1 };

__device__ __forceinline__ float fp8_max(int fmt) { return fmt == kFp8E5M2 ? 57344.f : 448.f; }

__device__ __forceinline__ float fp8_scale_from_amax(unsigned amax_bits, int fmt) {
  const float amax = __uint_as_float(amax_bits);
  return amax == 0.f ? 1.f : __fdiv_rn(amax, fp8_max(fmt));
}

// Division of many values by one scale s, correctly rounded like an IEEE fp32 division
// but with one reciprocal per scale: Markstein's division (the theorem that, with r the
// correctly rounded reciprocal of s and q = RN(y * r), the remainder y - q * s is exact
// in one fused multiply-add and RN(q + rem * r) is the correctly rounded quotient;
// P. Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34 (1990); Handbook of Floating-Point Arithmetic,
// Muller et al., chapter on division). It holds for normal s away from the ends of the
// range, which `ScaleDiv` checks once, falling back to __fdiv_rn. A zero remainder
// keeps q itself (and the sign of a zero quotient). The tests compare every code with
// a plain IEEE division.
struct ScaleDiv {
  float s, r;
  bool fast;
  __device__ __forceinline__ explicit ScaleDiv(float s_) : s(s_) {
    fast = s_ >= 0x1p-120f && s_ <= 0x1p120f;
    r = fast ? __frcp_rn(s_) : 1.f;
  }
  __device__ __forceinline__ float operator()(float y) const {
    if (!fast) return __fdiv_rn(y, s);
    const float q = __fmul_rn(y, r);
    const float rem = __fmaf_rn(-q, s, y);
    return rem == 0.f ? q : __fmaf_rn(rem, r, q);
  }
};

// two fp32 values -> two codes (low byte = v.x), round to nearest even, saturating
__device__ __forceinline__ unsigned short fp8x2(float2 v, int fmt) {
  return static_cast<unsigned short>(
      __nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, fmt == kFp8E5M2 ? __NV_E5M2 : __NV_E4M3));
}

}  // namespace moe
