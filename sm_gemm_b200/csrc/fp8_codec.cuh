// FP32 -> E4M3 group encoding shared by the quantiser (quant_fp8.cu) and the GEMM
// epilogue's FP8 output (epilogue.cuh): the group scale s = amax / 448 (1 for an
// all-zero group), the correctly rounded quotient x / s, and the round-to-nearest-even
// saturating conversion, following the DeepGEMM kernel-library walkthrough (zwxr.cn),
// section 2.4.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace smg {

__device__ __forceinline__ float group_scale(float amax) {
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

// Correctly rounded x / s for every element of a group that shares the scale s.
// Markstein's FMA division (P. Markstein, "IA-64 and Elementary Functions", 2000,
// chapter 8; also Muller et al., "Handbook of Floating-Point Arithmetic", the
// section on division with an FMA): with r = RN(1/s), y = RN(x r) and the residual
// e = x - y s (exact in one FMA), RN(y + e r) is the correctly rounded quotient
// provided r is the correctly rounded reciprocal and the significand of s is not
// all ones. The residual is exact only while x - y s stays out of the subnormal
// range, which holds for every quotient E4M3 can tell from zero (|x/s| > 2^-11)
// once s >= 2^-90; smaller quotients become a signed zero code either way, and
// the sign survives every step. A group whose scale fails a condition (all-ones
// significand, s < 2^-90, s not finite) divides with __fdiv_rn instead
// (ExactDiv); the choice is made once per group, outside the element loops.
__device__ __forceinline__ bool markstein_ok(float s) {
  const uint32_t b = __float_as_uint(s);
  const uint32_t ex = (b >> 23) & 0xffu;
  return ex >= 127u - 90u && ex < 255u && (b & 0x7fffffu) != 0x7fffffu;
}

struct MarksteinDiv {
  float s, r;  // r = RN(1 / s)
  // The residual step with e == 0 returns y + 0, which is +0 for x = -0: the sign of x
  // is ORed back in (a no-op for every other x, whose quotient already carries it).
  __device__ __forceinline__ float operator()(float x) const {
    const float y = __fmul_rn(x, r);
    const float e = __fmaf_rn(-y, s, x);
    const float q = __fmaf_rn(e, r, y);
    return __uint_as_float(__float_as_uint(q) | (__float_as_uint(x) & 0x80000000u));
  }
  // Two quotients with packed FP32x2 arithmetic (mul/fma.rn.f32x2; each half is
  // rounded exactly like the scalar operation).
  __device__ __forceinline__ float2 div2(float2 x) const {
    const float2 s2 = make_float2(s, s), r2 = make_float2(r, r);
    const float2 y = __fmul2_rn(x, r2);
    const float2 e = __ffma2_rn(make_float2(-y.x, -y.y), s2, x);
    const float2 q = __ffma2_rn(e, r2, y);
    return make_float2(__uint_as_float(__float_as_uint(q.x) | (__float_as_uint(x.x) & 0x80000000u)),
                       __uint_as_float(__float_as_uint(q.y) | (__float_as_uint(x.y) & 0x80000000u)));
  }
};

struct ExactDiv {
  float s;
  __device__ __forceinline__ float operator()(float x) const { return __fdiv_rn(x, s); }
};

__device__ __forceinline__ MarksteinDiv markstein_div(float s) { return MarksteinDiv{s, __frcp_rn(s)}; }

// Two codes packed little-endian: x0 -> low byte, x1 -> high byte.
__device__ __forceinline__ uint32_t e4m3x2(float x0, float x1) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3));
}

// Four codes of x[0..3] / s, little-endian in one word.
__device__ __forceinline__ uint32_t pack4(const MarksteinDiv& div, const float (&x)[4]) {
  const float2 a = div.div2(make_float2(x[0], x[1]));
  const float2 b = div.div2(make_float2(x[2], x[3]));
  return e4m3x2(a.x, a.y) | (e4m3x2(b.x, b.y) << 16);
}

__device__ __forceinline__ uint32_t pack4(const ExactDiv& div, const float (&x)[4]) {
  return e4m3x2(div(x[0]), div(x[1])) | (e4m3x2(div(x[2]), div(x[3])) << 16);
}

}  // namespace smg
