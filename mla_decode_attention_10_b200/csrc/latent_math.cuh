// latent_math.cuh -- element arithmetic of the latent rows (device side).
//
// bf16 <-> fp32, the rotate-half RoPE pair, the fp32 quotient x / scale and
// the packed e4m3 / bf16 conversions.  Every operation is written with
// explicitly rounded intrinsics so that the compiler cannot contract a
// product and a sum into one fused multiply-add: the results are the fp32
// values of the plain formulas, bit for bit.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace mla {

// bf16 bits -> fp32 (exact: bf16 is the top half of an fp32 word).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_bits(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

// Two fp32 -> packed bf16x2, round to nearest even; `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint16_t to_bf16(float v) {
  return static_cast<uint16_t>(pack_bf16x2(v, 0.0f) & 0xffffu);
}

// Two fp32 -> packed OCP E4M3FN pair, round to nearest even, saturating to
// +-448 (infinities included; NaN stays NaN); `lo` lands in bits 0..7.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Rotate-half RoPE of one pair: (a, b) -> (a c - b s, b c + a s), every
// product and sum rounded on its own.
__device__ __forceinline__ void rope_pair(float a, float b, float c, float s, float& ya, float& yb) {
  ya = __fsub_rn(__fmul_rn(a, c), __fmul_rn(b, s));
  yb = __fadd_rn(__fmul_rn(b, c), __fmul_rn(a, s));
}

// Per-tensor divisor.  `fast` holds when 2^-64 <= scale <= 2^64, where the
// corrected-reciprocal quotient below is exact; otherwise quotients go
// through the IEEE division intrinsic.
struct Divisor {
  float s;
  float y;  // reciprocal of s, rounded to nearest
  bool fast;
};

__device__ __forceinline__ Divisor make_divisor(float s) {
  Divisor d;
  d.s = s;
  d.fast = (s >= 0x1p-64f) && (s <= 0x1p64f);
  d.y = d.fast ? __frcp_rn(s) : 1.0f;
  return d;
}

// x / s rounded to nearest even in fp32 (the IEEE quotient), for `fast` s.
//
// Method (Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also Cornea, Harrison
// & Tang, "Scientific Computing on Itanium-based Systems", 2002): with
// y = RN(1/s) and a quotient estimate q, the residual r = x - q s is exact in
// one fused multiply-add whenever q is within an ulp of x/s, and
// RN(q + r y) is then the correctly rounded quotient.  q0 = RN(x y) can be
// up to ~1.5 ulp off, so one correction step first makes it faithful, and a
// second one rounds it correctly.  Zero keeps the sign of x (s > 0).  When
// |x y| is not below 2^126 (so that no correction step could overflow) or is
// infinite or NaN, q0 is returned as is: the e4m3 result saturates to 448 or
// is NaN whatever its last bits are.
// Below |x| ~ 2^-102 the residual may underflow and the last bits of the
// quotient may then differ from the IEEE quotient, but there |x / s| <= 2^-38,
// which every e4m3 rounding sends to the same signed zero.
__device__ __forceinline__ float div_rn(float x, const Divisor& d) {
  if (!d.fast) return __fdiv_rn(x, d.s);
  const float q0 = __fmul_rn(x, d.y);
  const float r0 = __fmaf_rn(-q0, d.s, x);
  const float q1 = __fmaf_rn(r0, d.y, q0);
  const float r1 = __fmaf_rn(-q1, d.s, x);
  const float q2 = __fmaf_rn(r1, d.y, q1);
  return fabsf(q0) < 0x1p126f ? copysignf(q2, x) : q0;
}

// Eight bf16 (one 16-byte chunk) -> eight e4m3 bytes of x / s.
__device__ __forceinline__ uint2 chunk_to_e4m3(const uint4 v, const Divisor& d) {
  uint2 o;
  const uint32_t p0 = pack_e4m3x2(div_rn(bf16_lo(v.x), d), div_rn(bf16_hi(v.x), d));
  const uint32_t p1 = pack_e4m3x2(div_rn(bf16_lo(v.y), d), div_rn(bf16_hi(v.y), d));
  const uint32_t p2 = pack_e4m3x2(div_rn(bf16_lo(v.z), d), div_rn(bf16_hi(v.z), d));
  const uint32_t p3 = pack_e4m3x2(div_rn(bf16_lo(v.w), d), div_rn(bf16_hi(v.w), d));
  o.x = p0 | (p1 << 16);
  o.y = p2 | (p3 << 16);
  return o;
}

}  // namespace mla
