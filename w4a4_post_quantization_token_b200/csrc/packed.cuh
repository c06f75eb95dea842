// Packed fp32x2 arithmetic (Blackwell f32x2 instructions): two IEEE fp32 lanes per
// 64-bit register, each lane rounded exactly like the scalar instruction.
#pragma once
#include <cstdint>

namespace kq {

__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ float f2lo(uint64_t r) { float a, b; f2unpack(r, a, b); return a; }
__device__ __forceinline__ float f2hi(uint64_t r) { float a, b; f2unpack(r, a, b); return b; }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fsub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// the two bf16 halves of a 32-bit word as an fp32 pair (exact)
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
  return f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Four E2M1 conversions (8 values, already divided by the block scale) packed into one
// 32-bit word, value 2j in the low nibble of byte j.
__device__ __forceinline__ uint32_t cvt_e2m1x8(uint64_t p0, uint64_t p1, uint64_t p2, uint64_t p3) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t.reg .f32 a0, a1, a2, a3, a4, a5, a6, a7;\n\t"
      "mov.b64 {a0, a1}, %1;\n\t"
      "mov.b64 {a2, a3}, %2;\n\t"
      "mov.b64 {a4, a5}, %3;\n\t"
      "mov.b64 {a6, a7}, %4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, a1, a0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, a3, a2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, a5, a4;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, a7, a6;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out) : "l"(p0), "l"(p1), "l"(p2), "l"(p3));
  return out;
}

}  // namespace kq
