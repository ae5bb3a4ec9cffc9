// mx.cuh -- MXFP8 conversion of 32 fp32 values (one block along K).
//
// CODA sparse-MoE thread (digg.com): the low-precision conversions of the
// expert GEMMs' inputs run in the epilogues of the kernels that produce them.
// Format: OCP Microscaling MXFP8 -- a block of 32 values shares the scale
// 2^e, e = floor(log2(max |v|)) - 8 (8 = exponent of E4M3's largest normal,
// 448), stored as the E8M0 byte e + 127 (clamped to [0, 254]; an all-zero
// block gets 0); each value is v * 2^-e rounded to nearest-even E4M3 with
// magnitudes above 448 clamped to 448 (cvt ... satfinite).
#pragma once

#include <cstdint>

namespace moe {

// E8M0 byte of a block whose largest magnitude is amax (amax >= 0).  For a
// normal float, floor(log2 amax) = exponent field - 127, so the byte is the
// exponent field - 8; zero and subnormal maxima give 0 (e = -127).
__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  const int ef = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  const int b = ef - 8;
  return b < 0 ? 0u : (b > 254 ? 254u : static_cast<uint32_t>(b));
}

// 2^(127 - byte) = 2^-e, exactly (float exponent field 254 - byte; byte 254
// gives the subnormal 2^-127).
__device__ __forceinline__ float mx_inv_scale(uint32_t byte) {
  return byte <= 253u ? __uint_as_float((254u - byte) << 23) : __uint_as_float(0x00400000u);
}

// Two fp32 -> two E4M3 (round to nearest even, saturating); lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// One MX block: 32 values -> 32 codes (8 words, value i in byte i % 4 of
// word i / 4) and the returned scale byte.
__device__ __forceinline__ uint32_t mx_quantize32(const float (&v)[32], uint32_t (&q)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb = mx_scale_byte(amax);
  const float inv = mx_inv_scale(sb);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    q[j] = e4m3x2(v[4 * j] * inv, v[4 * j + 1] * inv) | (e4m3x2(v[4 * j + 2] * inv, v[4 * j + 3] * inv) << 16);
  return sb;
}

}  // namespace moe
