// Block-scaled FP8 / FP4 storage of the caches ("DeepSeek V4 Inside", "What
// does HCA change?": BF16 on the K=V RoPE dims, FP8 on the others, FP4 for
// the indexer keys).  Element formats and block scaling follow the OCP
// Microscaling (MX) formats: 32 consecutive values share a power-of-two
// scale stored as E8M0 (exponent + 127), chosen as the smallest power of
// two that keeps the block's largest magnitude within the element format
// (E4M3: 448, E2M1: 6); elements are rounded to nearest even.
//
// Mixed K=V row (D dims, the last R in BF16):
//   bytes [0, D-R)              E4M3 codes of dims 0 .. D-R-1
//   bytes [D-R, D-R+2R)         BF16 of dims D-R .. D-1, as stored
//   bytes [D-R+2R, +(D-R)/32)   E8M0 scales, one per 32 dims
//   zero padding to a multiple of 16 bytes (592 at D = 512, R = 64)
// FP4 indexer keys: D/2 bytes of E2M1 codes per key (element 2i in the low
// nibble), and D/32 E8M0 scales per key in a separate array.
#pragma once

#include "ds4a_internal.cuh"

namespace ds4a {

constexpr int kMxBlock = 32;

__host__ __device__ constexpr int kv_fp8_row_bytes(int D, int R) {
  return ((D - R) + 2 * R + (D - R) / kMxBlock + 15) / 16 * 16;
}

// E8M0 scale code of a block whose largest magnitude is amax (>= 0): the
// smallest s with amax <= largest * 2^s, s in [-127, 127], as exponent + 127.
// amax = 1.m 2^(E-127) and largest = g 2^j with g = 0.875, j = 9 (E4M3,
// 448) or g = 0.75, j = 3 (E2M1, 6): s = E - 126 - j, plus one when the
// mantissa of amax exceeds that of the largest (1.m > 2g).
template <bool kFp4>
__device__ __forceinline__ int mx_scale_code(float amax) {
  const unsigned int bits = __float_as_uint(amax);
  const int E = (int)(bits >> 23);
  if (E == 0) return 0;  // zero or subnormal block maximum: s = -127
  const unsigned int mant = bits & 0x7FFFFFu;
  const int j = kFp4 ? 3 : 9;
  const unsigned int gm = kFp4 ? 0x400000u : 0x600000u;
  int s = E - 126 - j + (mant > gm ? 1 : 0);
  s = max(-127, min(127, s));
  return s + 127;
}

// 2^-(code - 127) as a float: the factor that maps the block into range
__device__ __forceinline__ float mx_inv_scale(int code) {
  const int e = 127 - (code - 127);  // biased exponent of 2^-(s)
  return e >= 1 ? __uint_as_float((unsigned int)e << 23) : __uint_as_float(0x00400000u >> (-e));
}

// 2^(code - 127) as a float (code 0 is 2^-127, a float subnormal)
__device__ __forceinline__ float mx_scale(int code) {
  return code >= 1 ? __uint_as_float((unsigned int)code << 23) : __uint_as_float(0x00400000u);
}

// two E4M3 codes (a in the low byte) of values already in range
__device__ __forceinline__ uint16_t to_e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

// two E2M1 codes packed in one byte (a in the low nibble)
__device__ __forceinline__ uint32_t to_e2m1x2(float a, float b) {
  uint32_t r;
  asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u32.u8 %0, t;\n}" : "=r"(r) : "f"(b), "f"(a));
  return r & 0xFFu;
}

// Two codes -> their two values as float32, exactly (the hardware unpacks to
// f16x2; every E4M3 / E2M1 value is exact in f16), low code first.
__device__ __forceinline__ float2 e4m3x2_to_f2(uint32_t two) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(two & 0xFFFFu)));
  float2 r;
  asm("{\n .reg .f16 lo, hi;\n mov.b32 {lo, hi}, %2;\n cvt.f32.f16 %0, lo;\n cvt.f32.f16 %1, hi;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(h2));
  return r;
}

__device__ __forceinline__ float2 e2m1x2_to_f2(uint32_t byte) {
  uint32_t h2;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h2) : "r"(byte & 0xFFu));
  float2 r;
  asm("{\n .reg .f16 lo, hi;\n mov.b32 {lo, hi}, %2;\n cvt.f32.f16 %0, lo;\n cvt.f32.f16 %1, hi;\n}"
      : "=f"(r.x), "=f"(r.y)
      : "r"(h2));
  return r;
}

// value of an E4M3 code (exact; 0x7F / 0xFF are NaN and never produced)
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  const uint32_t e = (code >> 3) & 15u, m = code & 7u;
  const float mag = e == 0 ? (float)m * 0.001953125f  // m 2^-9
                           : __uint_as_float(((e + 120u) << 23) | (m << 20));
  return (code & 0x80u) ? -mag : mag;
}

// value of an E2M1 code (exact)
__device__ __forceinline__ float e2m1_value(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  const float mag = e == 0 ? (float)m * 0.5f : __uint_as_float(((e + 126u) << 23) | (m << 22));
  return (code & 8u) ? -mag : mag;
}

}  // namespace ds4a
