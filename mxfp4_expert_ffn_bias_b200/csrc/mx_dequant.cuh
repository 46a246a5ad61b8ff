// MXFP4 -> 16-bit float conversion on the device.
//
// An MXFP4 block is 32 FP4 E2M1 codes (two per byte, element 2j in the low
// nibble of byte j) sharing one E8M0 scale byte s = 2^(s-127) (ZeroModels
// GPT-OSS docs, "MXFP4 experts": uint8 nibble blocks plus e8m0 scales; code
// values per the OCP MX v1.0 FP4 E2M1 definition).
#pragma once

#include <stdint.h>

// Eight consecutive elements (one 32-bit word of packed codes: 4 bytes) with
// scale byte s -> eight bf16 values, element order preserved (word j of the
// result holds elements 2j (low half) and 2j+1 (high half)).
//
// Exact for 2 <= s <= 252: E2M1 magnitudes have at most two significant bits,
// so v * 2^(s-127) is a normal bf16. The unscaled bf16 pattern of each code is
// looked up with byte permutes from two 8-entry tables (low and high byte of
// the bf16 of |v|), the sign bit is moved into place, and one bf16x2 multiply
// by 2^(s-127) (exponent field s) applies the scale.
__device__ __forceinline__ uint4 mx_dequant8_bf16(uint32_t w, uint32_t s) {
  // |v| for codes 0..7 = 0, .5, 1, 1.5, 2, 3, 4, 6 as bf16: 0000 3F00 3F80 3FC0 4000 4040 4080 40C0
  constexpr uint32_t kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;  // low bytes of codes 0-3, 4-7
  constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u;  // high bytes of codes 0-3, 4-7
  const uint32_t mag = w & 0x77777777u;                       // nibble selectors without sign bits
  const uint32_t magB = mag >> 16;
  const uint32_t loA = __byte_perm(kLo0, kLo1, mag), hiA = __byte_perm(kHi0, kHi1, mag);
  const uint32_t loB = __byte_perm(kLo0, kLo1, magB), hiB = __byte_perm(kHi0, kHi1, magB);
  uint32_t o0 = __byte_perm(loA, hiA, 0x5140);  // elements 0, 1
  uint32_t o1 = __byte_perm(loA, hiA, 0x7362);  // elements 2, 3
  uint32_t o2 = __byte_perm(loB, hiB, 0x5140);  // elements 4, 5
  uint32_t o3 = __byte_perm(loB, hiB, 0x7362);  // elements 6, 7
  // Signs: element 2j's sign is bit 8j+3 of w (bit 8j+7 of w<<4) and goes to bit 15;
  // element 2j+1's sign is bit 8j+7 of w and goes to bit 31.
  const uint32_t w4 = w << 4;
  o0 |= __byte_perm(w4, w, 0x4400) & 0x80008000u;
  o1 |= __byte_perm(w4, w, 0x5511) & 0x80008000u;
  o2 |= __byte_perm(w4, w, 0x6622) & 0x80008000u;
  o3 |= __byte_perm(w4, w, 0x7733) & 0x80008000u;
  const uint32_t sc = s * 0x00800080u;  // bf16x2 (2^(s-127), 2^(s-127))
  uint4 r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r.x) : "r"(o0), "r"(sc));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r.y) : "r"(o1), "r"(sc));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r.z) : "r"(o2), "r"(sc));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r.w) : "r"(o3), "r"(sc));
  return r;
}

// Four packed bytes -> four f16x2 words of the UNSCALED E2M1 values (exact in
// f16), with the sm_100a hardware FP4 converter. Word j holds byte j: its low
// nibble in the low half. The block scale is applied by the caller to fp32
// partial sums.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t& h0, uint32_t& h1, uint32_t& h2, uint32_t& h3) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
}

// acc += a.lo * b.lo + a.hi * b.hi on f16x2 operands with fp32 accumulation
// (two mixed-precision FMAs; the products of two f16 values are exact in fp32).
__device__ __forceinline__ void fma2_f16_f32(float& acc0, float& acc1, uint32_t a, uint32_t b) {
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %2;\n\t"
      "mov.b32 {b0, b1}, %3;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
      "fma.rn.f32.f16 %1, a1, b1, %1;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "r"(a), "r"(b));
}
