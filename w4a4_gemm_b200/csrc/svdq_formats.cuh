// svdq_formats.cuh -- device-side number formats and the per-group 4-bit
// quantizer of SVDQuant ("SVDQuant: Absorbing Outliers by Low-Rank Components
// for 4-Bit Diffusion Models", Sec. 3, groups of Sec. 5.1).
//
// The quantizer decisions are taken in fp32 exactly as follows:
//   amax  = max |v|                         (exact)
//   s32   = amax / q_max                    (IEEE fp32 division, q_max = 6 or 7)
//   scale = E4M3(s32) saturating at 448     (NVFP4, round to nearest even)
//         | fp16(min(s32, 65504))           (INT4, round to nearest even)
//   q     = v * RN(1 / scale)               (IEEE reciprocal, one RN multiply)
//   code  = E2M1(q) saturating at 6, nearest even   (NVFP4)
//         | clamp(rint_even(q), -7, 7)               (INT4)
//   a zero scale yields all-zero codes.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace svdq {

// FP8 E4M3 code of a non-negative fp32 value, nearest even, saturating.
__device__ __forceinline__ uint32_t e4m3_code(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}

// Value of a non-negative finite E4M3 code, built from its bit fields
// (exponent bias 7, 3 mantissa bits; exponent field 0 = subnormal, m * 2^-9).
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  if (e == 0) return static_cast<float>(m) * (1.0f / 512.0f);
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eight fp32 values -> eight packed E2M1 codes (value 2i in the low nibble of
// byte i), nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t e2m1_pack8(const float* q) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(q[0]), "f"(q[1]), "f"(q[2]), "f"(q[3]), "f"(q[4]), "f"(q[5]), "f"(q[6]), "f"(q[7]));
  return out;
}

// NVFP4 group of 16 values (already smoothed): writes the 8 code bytes into
// codes[0..1] (two 32-bit words) and returns the E4M3 scale code.
__device__ __forceinline__ uint32_t quant16_nvfp4(const float* v, uint32_t* codes) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const float s32 = __fdiv_rn(amax, 6.0f);
  const uint32_t s8 = e4m3_code(s32);
  const float sd = e4m3_value(s8);
  if (sd == 0.0f) {
    codes[0] = 0u;
    codes[1] = 0u;
    return s8;
  }
  const float inv = __frcp_rn(sd);
  float q[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) q[i] = __fmul_rn(v[i], inv);
  codes[0] = e2m1_pack8(q);
  codes[1] = e2m1_pack8(q + 8);
  return s8;
}

// INT4 scale of a group whose absolute maximum is `amax`: fp16 bits.
__device__ __forceinline__ uint16_t int4_scale_bits(float amax) {
  const float s32 = __fdiv_rn(amax, 7.0f);
  return __half_as_ushort(__float2half_rn(fminf(s32, 65504.0f)));
}

// Signed INT4 code of one smoothed value given the decoded scale's reciprocal.
__device__ __forceinline__ int int4_code(float v, float inv) {
  int q = __float2int_rn(__fmul_rn(v, inv));
  return max(-7, min(7, q));
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

}  // namespace svdq
