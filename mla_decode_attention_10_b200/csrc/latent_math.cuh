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

// Per-tensor divisor.  `fast` holds when 2^-64 <= scale <= 2^64: there the
// quotients come from the corrected reciprocal below; otherwise (zero,
// negative, huge, tiny, NaN scales) from the IEEE division intrinsic.
struct Divisor {
  uint64_t s2;       // {s, s}
  uint64_t ny2;      // {-RN(1/s), -RN(1/s)}
  float s;
  float nclamp;      // -B, B = smallest power of two >= 512 s
  uint32_t nclamp2;  // -B as a bf16x2 pair (exact: B is a power of two)
  bool fast;
};

// {v, v} as one 64-bit operand of the packed f32x2 instructions.
__device__ __forceinline__ uint64_t pair_of(float v) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %1};" : "=l"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ Divisor make_divisor(float s) {
  Divisor d;
  d.s = s;
  d.fast = (s >= 0x1p-64f) && (s <= 0x1p64f);
  d.s2 = pair_of(s);
  d.ny2 = pair_of(d.fast ? -__frcp_rn(s) : -1.0f);
  uint32_t b = __float_as_uint(d.fast ? 512.0f * s : 1.0f);
  b = (b & 0x007fffffu) ? ((b & 0x7f800000u) + 0x00800000u) : b;
  d.nclamp = -__uint_as_float(b);
  const uint32_t hb = __float_as_uint(d.nclamp) >> 16;
  d.nclamp2 = hb | (hb << 16);
  return d;
}

// -min(|x|, B) with the sign of x flipped; NaN stays NaN.  Values beyond B
// divide to more than 512 and saturate to 448 in e4m3 whatever they are, so
// the clamp changes no e4m3 result and keeps the quotient below 1024.
__device__ __forceinline__ float neg_clamp(float x, const Divisor& d) {
  float m;
  asm("min.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(m) : "f"(x), "f"(d.nclamp));
  return m;
}

// Same on a bf16x2 pair (both halves at once).
__device__ __forceinline__ uint32_t neg_clamp_bf16x2(uint32_t w, const Divisor& d) {
  uint32_t m;
  asm("min.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(m) : "r"(w), "r"(d.nclamp2));
  return m;
}

// Quotients x / s of two values given as mx = -x (after neg_clamp), rounded
// to nearest even in fp32, two lanes of fp32 arithmetic per instruction
// (packed f32x2 multiply and fused multiply-add of sm_100).
//
// Method (Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also Cornea, Harrison
// & Tang, "Scientific Computing on Itanium-based Systems", 2002): with
// y = RN(1/s) and a quotient estimate q within an ulp of x/s, the residual
// r = x - q s is exact in one fused multiply-add and RN(q + r y) is the
// correctly rounded quotient.  q0 = RN(x y) can be up to ~1.5 ulp off, so a
// first correction makes it faithful and a second rounds it correctly.  The
// steps are written on -x and -y so that every operand enters the FMA
// unnegated: q0 = (-x)(-y), r = q s + (-x), q <- r (-y) + q; with these
// forms a zero x gives a zero quotient of the same sign.  Below |x| ~ 2^-100
// the residual may underflow and the last bits may differ from the IEEE
// quotient, but there |x / s| <= 2^-36, which every e4m3 rounding sends to
// the same signed zero.
__device__ __forceinline__ void quotient_pair_neg(float mlo, float mhi, const Divisor& d, float& qlo,
                                                  float& qhi) {
  asm("{\n\t"
      ".reg .b64 mx, q, r;\n\t"
      "mov.b64 mx, {%2, %3};\n\t"
      "mul.rn.f32x2 q, mx, %5;\n\t"
      "fma.rn.f32x2 r, q, %4, mx;\n\t"
      "fma.rn.f32x2 q, r, %5, q;\n\t"
      "fma.rn.f32x2 r, q, %4, mx;\n\t"
      "fma.rn.f32x2 q, r, %5, q;\n\t"
      "mov.b64 {%0, %1}, q;\n\t"
      "}"
      : "=f"(qlo), "=f"(qhi)
      : "f"(mlo), "f"(mhi), "l"(d.s2), "l"(d.ny2));
}

// e4m3 bytes of lo / s and hi / s for two fp32 values (lo in bits 0..7).
// FAST: the divisor's scale is in [2^-64, 2^64] (d.fast), decided once per
// kernel so that the per-element code has no branch.
template <bool FAST>
__device__ __forceinline__ uint32_t e4m3x2_of_f32(float lo, float hi, const Divisor& d) {
  float qlo, qhi;
  if (FAST) {
    quotient_pair_neg(neg_clamp(lo, d), neg_clamp(hi, d), d, qlo, qhi);
  } else {
    qlo = __fdiv_rn(lo, d.s);
    qhi = __fdiv_rn(hi, d.s);
  }
  return pack_e4m3x2(qlo, qhi);
}

// One corrected step of the quotient above: q0 = RN(x y), q1 = RN(q0 + r y).
// q1 may differ from the IEEE quotient in its last bit, but when x is a bf16
// value (8 significant bits) it has the same e4m3 byte.  Let z = x / s.
// q0 + r y = z + (z - q0)(s y - 1) with |s y - 1| <= 2^-24 and
// |z - q0| < 2 ulp(z), so it lies within 2^-23 ulp(z) of z.  Two adjacent
// fp32 values round to different e4m3 bytes only when one of them is an
// e4m3 rounding midpoint M (odd significand M' of at most 5 bits), so the
// bytes of q1 and RN(z) can differ only if z lies that close to a point
// m = M +- (half the fp32 spacing on that side of M).  In units of
// ulp(s) ulp(z) / 2, s m is the integer S (M' 2^k +- 1), with S the 24-bit
// significand of s and 20 <= k <= 25, and x would lie within 4 units of it.
// Modulo 2^k that forces S = c 2^k + r with |r| < 4, and then
// S (M' 2^k +- 1) = c M' 2^2k + (+-c + r M') 2^k +- r spans more than 8
// significant bits unless +-c + r M' = 0.  The only such case is
// M = 2^-10, S = 2^24 - 1 (s just below a power of two), where evaluating
// the two steps exactly gives q1 = RN(z).
__device__ __forceinline__ void quotient_pair_neg1(float mlo, float mhi, const Divisor& d, float& qlo,
                                                   float& qhi) {
  asm("{\n\t"
      ".reg .b64 mx, q, r;\n\t"
      "mov.b64 mx, {%2, %3};\n\t"
      "mul.rn.f32x2 q, mx, %5;\n\t"
      "fma.rn.f32x2 r, q, %4, mx;\n\t"
      "fma.rn.f32x2 q, r, %5, q;\n\t"
      "mov.b64 {%0, %1}, q;\n\t"
      "}"
      : "=f"(qlo), "=f"(qhi)
      : "f"(mlo), "f"(mhi), "l"(d.s2), "l"(d.ny2));
}

// e4m3 bytes of the two bf16 of `w` divided by s (low half in bits 0..7).
// FAST takes the one-step quotient (exact in e4m3 for bf16 inputs, above).
template <bool FAST>
__device__ __forceinline__ uint32_t e4m3x2_of_bf16x2(uint32_t w, const Divisor& d) {
  float qlo, qhi;
  if (FAST) {
    const uint32_t m = neg_clamp_bf16x2(w, d);
    quotient_pair_neg1(bf16_lo(m), bf16_hi(m), d, qlo, qhi);
  } else {
    qlo = __fdiv_rn(bf16_lo(w), d.s);
    qhi = __fdiv_rn(bf16_hi(w), d.s);
  }
  return pack_e4m3x2(qlo, qhi);
}

// Eight bf16 (one 16-byte chunk) -> eight e4m3 bytes of x / s.
template <bool FAST>
__device__ __forceinline__ uint2 chunk_to_e4m3(const uint4 v, const Divisor& d) {
  uint2 o;
  o.x = e4m3x2_of_bf16x2<FAST>(v.x, d) | (e4m3x2_of_bf16x2<FAST>(v.y, d) << 16);
  o.y = e4m3x2_of_bf16x2<FAST>(v.z, d) | (e4m3x2_of_bf16x2<FAST>(v.w, d) << 16);
  return o;
}

}  // namespace mla
