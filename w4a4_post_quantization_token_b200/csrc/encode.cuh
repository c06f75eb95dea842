// MXFP4 encoding of one 32-element block held in registers (OCP Microscaling
// Formats v1.0 rule, the format the KroQuant commentary, section 03, quantizes to):
//   e     = clamp(floor(log2(amax)) - 2, -127, 127), scale byte = e + 127
//   code  = round-to-nearest-even of v / 2^e on the E2M1 grid, saturated at +-6,
//           sign bit taken from v.
// floor(log2(amax)) comes from the float32 exponent field; for a subnormal amax
// the clamp already gives e = -127, so no leading-zero count is needed. The scaling
// by 2^-e is an exact power-of-two multiply (the build keeps denormals, no FTZ).
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace kq {

// Pack two floats into one byte of E2M1 codes: `lo` in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\t"
      "cvt.u32.u8 %0, b;\n\t}"
      : "=r"(out) : "f"(hi), "f"(lo));
  return out;
}

// Shared exponent byte (e + 127) of a block with maximum magnitude amax.
__device__ __forceinline__ uint32_t mx_scale_byte(float amax) {
  const int be = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu);
  return static_cast<uint32_t>(max(be - 2, 0));    // (be - 127) - 2 + 127, clamped at e = -127
}

// 2^-e for a scale byte sb = e + 127, as an exact float (e in [-127, 125] here).
__device__ __forceinline__ float mx_inv_scale(uint32_t sb) {
  return __uint_as_float((254u - sb) << 23);     // exponent field 127 - e = 254 - sb
}

// Encode v[0..31] (already in registers). Writes 16 bytes of packed codes (element 2j
// in the low nibble of byte j) into c[0..3] and returns the scale byte.
__device__ __forceinline__ uint32_t mx_encode32(const float (&v)[32], uint32_t (&c)[4]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb = mx_scale_byte(amax);
  const float inv = mx_inv_scale(sb);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e0 = 8 * w + 2 * j;
      word |= cvt_e2m1x2(v[e0] * inv, v[e0 + 1] * inv) << (8 * j);
    }
    c[w] = word;
  }
  return sb;
}

// Codes of v[0..31] at a given scale byte (same rounding as mx_encode32).
__device__ __forceinline__ void mx_codes_at(const float (&v)[32], uint32_t sb, uint32_t (&c)[4]) {
  const float inv = mx_inv_scale(sb);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e0 = 8 * w + 2 * j;
      word |= cvt_e2m1x2(v[e0] * inv, v[e0 + 1] * inv) << (8 * j);
    }
    c[w] = word;
  }
}

// Robust l_p fit of the block scale (CentriQ: weights fitted under an l_p objective that
// tracks each group's dense mode and discounts heavy tails). Candidates: the OCP byte sb0
// and sb0 - 1 .. sb0 - 3 (not below 0); codes as mx_encode32 at each; objective
// sum_k |v_k - deq_k|^p in float64, summed in element order; the smallest wins, ties keep
// the larger scale. Returns the scale byte, writes the codes.
__device__ __forceinline__ uint32_t mx_encode32_lp(const float (&v)[32], double p, uint32_t (&c)[4]) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const uint32_t sb0 = mx_scale_byte(amax);
  const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  uint32_t best_sb = sb0;
  double best_f = 0.0;
  for (int d = 0; d <= 3; ++d) {
    const uint32_t sb = sb0 >= static_cast<uint32_t>(d) ? sb0 - d : 0u;
    uint32_t cc[4];
    mx_codes_at(v, sb, cc);
    const double sc = ldexp(1.0, static_cast<int>(sb) - 127);
    double f = 0.0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const uint32_t code = (cc[k / 8] >> (4 * (k % 8))) & 0xFu;
      const double q = ((code & 8u) ? -mag[code & 7u] : mag[code & 7u]) * sc;
      const double err = fabs(static_cast<double>(v[k]) - q);
      f += (p == 1.0) ? err : (p == 2.0) ? err * err : pow(err, p);
    }
    if (d == 0 || f < best_f) {
      best_f = f;
      best_sb = sb;
#pragma unroll
      for (int w = 0; w < 4; ++w) c[w] = cc[w];
    }
  }
  return best_sb;
}

}  // namespace kq
