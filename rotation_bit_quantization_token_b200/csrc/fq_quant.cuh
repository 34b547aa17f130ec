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
  int mode;            // MxCase
  float dst_max;       // D = float32(dstTypeMax), the divisor of the ratio rule
  float inv_dst;       // float32(1 / D)
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
// Case-3 byte for a group whose q = fp32(amax * fp32(1 / D)) (exponent field Eq, mantissa
// field Mq) lies within 4 ulp of a power of two 2^k, is subnormal, or is not finite. With
// S = amax / D rounded to nearest in float32: S <= 2^k exactly when amax / D <= 2^k (1 +
// 2^-24) (the midpoint above 2^k rounds to 2^k, the even neighbour), i.e. when amax - D 2^k
// <= D 2^(k - 24). amax and D 2^k are within a factor two of each other, so one FMA gives
// their difference exactly (Sterbenz). For k >= -125 the byte is then k + 127 when S <= 2^k
// (S in (2^(k-1), 2^k]: exponent k - 1 plus one, or 2^k itself) and k + 128 otherwise. A
// non-finite amax gets 255, the byte the rule gives an infinite or NaN S.
__device__ __forceinline__ uint32_t ratio_byte_exact(float amax, float D, uint32_t Eq, uint32_t Mq) {
  if (Eq >= 254u) return 255u;
  const int k = Eq == 0u ? -126 : (Mq <= 3u ? int(Eq) - 127 : int(Eq) - 126);  // 2^k next to q
  if (k <= -126) {
    // S near 2^-126, the bottom of the normal range: a subnormal S gives 0, S = 2^-126 gives
    // 1 (mantissa 0), S above it 2. S > 2^-126 exactly when amax - D 2^-126 > D 2^-150, and
    // S >= 2^-126 when amax - D 2^-126 >= -D 2^-150 (the midpoint below 2^-126 rounds up,
    // to the even neighbour). Scaled by 2^64 (exact) every term is a normal float.
    const float a = amax * __uint_as_float(uint32_t(127 + 64) << 23);
    const float r = fmaf(-D, __uint_as_float(uint32_t(127 - 62) << 23), a);
    const float t = D * __uint_as_float(uint32_t(127 - 86) << 23);
    return r > t ? 2u : (r >= -t ? 1u : 0u);
  }
  const float p = __uint_as_float(uint32_t(k + 127) << 23);
  const float r = fmaf(-D, p, amax);
  // D 2^(k - 24), exact: k >= -125 keeps 2^(k - 24) at 2^-149 or above, and the product is
  // formed in two steps when 2^(k - 24) is below the normal range
  const float t = k - 24 >= -126
                      ? D * __uint_as_float(uint32_t(k + 127 - 24) << 23)
                      : (D * __uint_as_float(uint32_t(k + 127 + 40) << 23)) * __uint_as_float(uint32_t(127 - 64) << 23);
  return r <= t ? uint32_t(k + 127) : uint32_t(k + 128);
}

// E8M0 byte of one group from its float32 absolute maximum, by the common path of each rule
// (see mx_scale); for the ratio rule *rare is set when the byte must instead be decided by
// mx_byte_rare (q within 4 ulp of a power of two, subnormal, or amax not finite).
//  case 1 (0.0):     e = floor(log2 amax) - 2, clamped to [-127, 127]
//  case 2 (6.0/7.0): e = floor(log2 amax) - 2 + [leading one/two fraction bits set and
//                    the remaining fraction bits not all zero]
//  case 3 (other):   S = fp32(amax / dstTypeMax); E = biased exponent of S, plus one
//                    when S is normal, E < 254 and S's mantissa field is nonzero.
// For the first two cases a zero or subnormal amax always clamps to e = -127 (byte 0).
template <int kOnly = 0>  // kMxRatio: compiled for the ratio rule alone; 0: any rule
__device__ __forceinline__ uint32_t mx_byte_common(float amax, MxRule rule, bool* rare) {
  if (kOnly == kMxRatio || rule.mode == kMxRatio) {
    // q = amax * fp32(1 / D) is within 2.5 ulp of S = fp32(amax / D): when q's exponent field
    // is in [1, 253] and its mantissa field in [4, 2^23 - 5], S has q's exponent and a
    // nonzero mantissa, so the byte is q's exponent field plus one
    const uint32_t qb = __float_as_uint(amax * rule.inv_dst);
    const uint32_t Eq = (qb >> 23) & 0xFFu, Mq = qb & 0x7FFFFFu;
    *rare = Eq - 1u >= 253u || Mq - 4u > 0x7FFFFAu - 4u;
    return Eq + 1u;
  }
  *rare = false;
  const uint32_t bits = __float_as_uint(amax);
  const uint32_t Ef = (bits >> 23) & 0xFFu;
  if (Ef == 0u) return 0u;  // zero or subnormal: e = -127
  int e = int(Ef) - 127 - 2;
  const uint32_t frac = bits & 0x7FFFFFu;
  if (rule.mode == kMxMantissa6) e += (frac > 0x400000u) ? 1 : 0;
  else if (rule.mode == kMxMantissa7) e += (frac > 0x600000u) ? 1 : 0;
  e = e < -127 ? -127 : e;  // floor(log2 amax) >= -126 here, so only the low clamp binds
  return uint32_t(e + 127);
}

// The ratio-rule byte of a group that mx_byte_common marked rare, decided exactly.
__device__ __forceinline__ uint32_t mx_byte_rare(float amax, MxRule rule) {
  const uint32_t qb = __float_as_uint(amax * rule.inv_dst);
  return ratio_byte_exact(amax, rule.dst_max, (qb >> 23) & 0xFFu, qb & 0x7FFFFFu);
}

// Byte and the exact power-of-two multiplier R of one group (each element is encoded as
// E2M1(x * R)), for a caller that decides each lane on its own.
__device__ __forceinline__ MxScale mx_scale(float amax, MxRule rule) {
  bool rare;
  MxScale s;
  s.byte = mx_byte_common(amax, rule, &rare);
  if (rare) s.byte = mx_byte_rare(amax, rule);
  s.R = pow2_from_e8m0_inverse_any(s.byte);
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
