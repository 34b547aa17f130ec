// Device-side quantizer arithmetic shared by both kernels of libfq.
//
// Page: "aclnnFlatQuantV2 complete guide: from two-level matmul to FP4 E2M1
// quantization fusion" (http://www.zwxr.cn/news/277566), "per-token mode" and
// "per-group mode" cases 1-3. All decisions (codes, exponents) are taken in float32
// from the float32 value of x''.
#pragma once

#include <cstdint>

namespace fq {

// Per-group rule selected by dstTypeMax.
enum MxCase : int { kMxFloor = 1, kMxMantissa6 = 2, kMxMantissa7 = 3, kMxRatio = 4 };

struct MxRule {
  int mode;        // MxCase
  float dst_max;   // float32(dstTypeMax) for the ratio rule
  float inv_dst;   // float32(1 / dstTypeMax), used by the tensor-core kernel
};

// E8M0 byte and the exact power-of-two multiplier R such that each element of the
// group is encoded as E2M1(x * R).
struct MxScale {
  uint32_t byte;
  float R;
};

// 2^(127 - b) as float32 for a biased exponent b in [0, 253] (always a normal number).
__device__ __forceinline__ float pow2_from_e8m0_inverse(uint32_t b) {
  return __uint_as_float((254u - b) << 23);
}

// The same for every byte the ratio rule can give: 254 is 2^-127 (a subnormal), and 255,
// the byte of a non-finite S, gets 0 (1 / infinity), so no byte wraps the exponent field.
__device__ __forceinline__ float pow2_from_e8m0_inverse_any(uint32_t b) {
  return b <= 253u ? pow2_from_e8m0_inverse(b) : (b == 254u ? __uint_as_float(0x00400000u) : 0.0f);
}

// Shared exponent of one group from its float32 absolute maximum.
//  case 1 (0.0):     e = floor(log2 amax) - 2, clamped to [-127, 127]
//  case 2 (6.0/7.0): e = floor(log2 amax) - 2 + [leading one/two fraction bits set and
//                    the remaining fraction bits not all zero]
//  case 3 (other):   S = fp32(amax / dstTypeMax); E = biased exponent of S, plus one
//                    when S is normal, E < 254 and S's mantissa field is nonzero.
// For the first two cases a zero or subnormal amax always clamps to e = -127 (byte 0).
template <bool kExactDiv = true>
__device__ __forceinline__ MxScale mx_scale(float amax, MxRule rule) {
  MxScale s;
  if (rule.mode == kMxRatio) {
    // S = amax / dstTypeMax in float32, rounded to nearest (both kernels). kExactDiv =
    // false would multiply by the float32 reciprocal instead: within one ulp of the
    // quotient, which can move the byte when amax / dstTypeMax is a power of two.
    const float S = kExactDiv ? __fdiv_rn(amax, rule.dst_max) : amax * rule.inv_dst;
    const uint32_t bits = __float_as_uint(S);
    uint32_t E = (bits >> 23) & 0xFFu;
    const uint32_t mant = bits & 0x7FFFFFu;
    if (E >= 1u && E < 254u && mant != 0u) E += 1u;
    s.byte = E;
    s.R = pow2_from_e8m0_inverse_any(E);  // E is 255 only for a non-finite S
    return s;
  }
  const uint32_t bits = __float_as_uint(amax);
  const uint32_t Ef = (bits >> 23) & 0xFFu;
  if (Ef == 0u) {  // zero or subnormal: e = -127
    s.byte = 0u;
    s.R = pow2_from_e8m0_inverse(0u);
    return s;
  }
  int e = int(Ef) - 127 - 2;
  const uint32_t frac = bits & 0x7FFFFFu;
  if (rule.mode == kMxMantissa6) e += (frac > 0x400000u) ? 1 : 0;
  else if (rule.mode == kMxMantissa7) e += (frac > 0x600000u) ? 1 : 0;
  e = e < -127 ? -127 : e;  // floor(log2 amax) >= -126 here, so only the low clamp binds
  s.byte = uint32_t(e + 127);
  s.R = pow2_from_e8m0_inverse(s.byte);
  return s;
}

// Two E2M1 codes (round to nearest even, saturate to +-6) packed in one byte: `lo` in
// bits 0-3, `hi` in bits 4-7. The hardware conversion keeps the sign of values that round
// to zero; e2m1_canonical_zero() removes it.
__device__ __forceinline__ uint32_t e2m1x2_raw(float lo, float hi) {
  uint16_t r;
  // The first source operand lands in the upper nibble, the second in the lower.
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u16.u8 %0, t;\n\t}"
      : "=h"(r)
      : "f"(hi), "f"(lo));
  return uint32_t(r) & 0xFFu;
}

// Clears the sign bit of every E2M1 nibble whose magnitude is zero (eight nibbles per
// word): a zero code is always +0 (0x0). For a nibble n, (n & 7) + 7 sets bit 3 exactly
// when the magnitude is nonzero, with no carry into the next nibble.
__device__ __forceinline__ uint32_t e2m1_canonical_zero(uint32_t w) {
  const uint32_t nonzero = ((w & 0x77777777u) + 0x77777777u) & 0x88888888u;
  return w & (0x77777777u | nonzero);
}

// INT4 code: round half to even, clamp to [-8, 7], as a 4-bit two's complement nibble.
__device__ __forceinline__ uint32_t int4_nibble(float v) {
  int q = __float2int_rn(v);
  q = q < -8 ? -8 : (q > 7 ? 7 : q);
  return uint32_t(q) & 0xFu;
}

// quantScale = fp32(amax / (7 / clipRatio)), the division taken in double.
__device__ __forceinline__ float per_token_scale(float amax, double clip_ratio) {
  return float(double(amax) / (7.0 / clip_ratio));
}

}  // namespace fq
