// svdq_formats.cuh -- device-side number formats and the per-group 4-bit
// quantizer of SVDQuant ("SVDQuant: Absorbing Outliers by Low-Rank Components
// for 4-Bit Diffusion Models", Sec. 3, groups of Sec. 5.1).
//
// The quantizer decisions are taken in fp32 exactly as follows:
//   amax  = max |v|                         (exact)
//   s32   = amax / q_max                    (IEEE fp32 quotient, q_max = 6 or 7)
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

// Value of an E2M1 code from its bit fields: sign bit 3, exponent bits 2..1
// (bias 1), mantissa bit 0; exponent field 0 = subnormal m * 0.5.
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? 0.5f * static_cast<float>(m)
                           : static_cast<float>(1u << (e - 1)) * (1.0f + 0.5f * static_cast<float>(m));
  return (code & 8u) ? -mag : mag;
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

// IEEE fp32 x / 6 and x / 7 without a division: q0 = x * RN(1/d),
// r = fma(-d, q0, x) (exact remainder), q = fma(r, RN(1/d), q0) -- the FMA
// division by a constant of Markstein and of Brisebarre & Muller ("Accelerating
// correctly rounded floating-point division when the divisor is known in
// advance", IEEE TC 2004).  Checked over every significand of a normal binade
// (and, by power-of-two scaling, every normal x) against IEEE division: equal
// for d = 7 everywhere and for d = 6 whenever x >= 2^-125; below that x / 6
// is subnormal and both round to the E4M3 scale 0.
__device__ __forceinline__ float div_by_const_rn(float x, float d, float rcp_d) {
  const float q0 = __fmul_rn(x, rcp_d);
  const float r = __fmaf_rn(-d, q0, x);
  return __fmaf_rn(r, rcp_d, q0);
}
__device__ __forceinline__ float div6_rn(float x) {
  return div_by_const_rn(x, 6.0f, __uint_as_float(0x3E2AAAABu));   // RN(1/6)
}
__device__ __forceinline__ float div7_rn(float x) {
  return div_by_const_rn(x, 7.0f, __uint_as_float(0x3E124925u));   // RN(1/7)
}

// Two fp32 products in one instruction (IEEE round-to-nearest per lane).
__device__ __forceinline__ float2 fmul2_rn(float2 a, float2 b) {
  unsigned long long x, y, z;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(y) : "f"(b.x), "f"(b.y));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(z) : "l"(x), "l"(y));
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(z));
  return r;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float m;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(a), "f"(b), "f"(c));
  return m;
}

// max |v_i| over 16 values
__device__ __forceinline__ float absmax16(const float* v) {
  const float a = fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
  const float b = fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
  const float c = fmax3(fabsf(v[6]), fabsf(v[7]), fabsf(v[8]));
  const float d = fmax3(fabsf(v[9]), fabsf(v[10]), fabsf(v[11]));
  const float e = fmax3(fabsf(v[12]), fabsf(v[13]), fabsf(v[14]));
  return fmax3(fmax3(a, b, c), fmax3(d, e, fabsf(v[15])), 0.0f);
}

// NVFP4 group of 16 values (already smoothed): writes the 8 code bytes into
// codes[0..1] (two 32-bit words) and returns the E4M3 scale code.  `rcp_tab`
// holds RN(1 / value) of every finite E4M3 code (0 for code 0).
__device__ __forceinline__ uint32_t quant16_nvfp4(const float* v, uint32_t* codes,
                                                  const float* rcp_tab) {
  const float s32 = div6_rn(absmax16(v));
  const uint32_t s8 = e4m3_code(s32);
  const float inv = rcp_tab[s8];
  if (inv == 0.0f) {               // zero scale: all codes 0
    codes[0] = 0u;
    codes[1] = 0u;
    return s8;
  }
  float q[16];
  const float2 i2 = make_float2(inv, inv);
#pragma unroll
  for (int i = 0; i < 16; i += 2) {
    const float2 r = fmul2_rn(make_float2(v[i], v[i + 1]), i2);
    q[i] = r.x;
    q[i + 1] = r.y;
  }
  codes[0] = e2m1_pack8(q);
  codes[1] = e2m1_pack8(q + 8);
  return s8;
}

// FP4 group of 32 values (one E4M3 scale for all 32): writes 16 code bytes
// into codes[0..3] and returns the E4M3 scale code.
__device__ __forceinline__ uint32_t quant32_fp4(const float* v, uint32_t* codes,
                                                const float* rcp_tab) {
  const float s32 = div6_rn(fmaxf(absmax16(v), absmax16(v + 16)));
  const uint32_t s8 = e4m3_code(s32);
  const float inv = rcp_tab[s8];
  float q[32];
  const float2 i2 = make_float2(inv, inv);
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float2 r = fmul2_rn(make_float2(v[i], v[i + 1]), i2);
    q[i] = r.x;
    q[i + 1] = r.y;
  }
#pragma unroll
  for (int w = 0; w < 4; ++w) codes[w] = inv == 0.0f ? 0u : e2m1_pack8(q + 8 * w);   // zero scale: zero codes
  return s8;
}

// Fill a 128-entry table with RN(1 / E4M3 value) for codes 0..127 (code 0 -> 0,
// NaN code 0x7F -> 0; scales never take it: they saturate at 448).
__device__ __forceinline__ void fill_e4m3_rcp_table(float* tab, int tid, int nthreads) {
  for (int c = tid; c < 128; c += nthreads) {
    const float v = e4m3_value(static_cast<uint32_t>(c));
    tab[c] = (c == 0 || c == 0x7F) ? 0.0f : __frcp_rn(v);
  }
}

// INT4 scale of a group whose absolute maximum is `amax`: fp16 bits.
__device__ __forceinline__ uint16_t int4_scale_bits(float amax) {
  const float s32 = div7_rn(amax);
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
