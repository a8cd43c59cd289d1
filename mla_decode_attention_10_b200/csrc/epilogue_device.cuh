// epilogue_device.cuh -- launch arguments and device helpers shared by the
// epilogue's kernels (internal).
//
// Rows of one call: rows [0, T) are the T cache rows (token t = row), rows
// [T, T + T*H) the query rows in q_out order (q = row - T, t = q / H,
// h = q % H).  Every row is 576 = 512 nope + 64 pe values wide; the pe part
// is rotated as 32 pairs (i, i + 32) (vLLM PR #54896 report, 实现拆解 items
// 1-3 and the writeLatent576 listing).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "latent_math.cuh"
#include "mla_epilogue.h"

namespace mla {

constexpr int kNope = 512;
constexpr int kPe = 64;
constexpr int kHalfPe = 32;
constexpr int kRow = 576;

struct Args {
  const uint16_t* q_nope;
  int64_t qn_st, qn_sh;
  const uint16_t* q_pe;
  int64_t qp_st, qp_sh;
  const uint16_t* kv_c;
  int64_t kv_st;
  const uint16_t* k_pe;
  int64_t kp_st;
  const int64_t* slots;
  const int32_t* positions;
  const float* cos_sin;
  int64_t rope_rows;
  const float* q_scale;
  const float* kv_scale;
  int64_t T;
  int64_t H;
  uint64_t h_magic;   // ceil(2^64 / H) for H >= 2, see div_heads
  uint32_t h_magic32;  // ceil(2^(31+s) / H), 2^(s-1) < H <= 2^s, for H >= 2; 0 for H = 1
  uint32_t h_shift32;  // s - 1
  int32_t pe_vec;      // q_pe / k_pe rows 4-byte aligned and the table 8-byte aligned: pe pairs two at a time
  int64_t cache_rows;
  int64_t rows;  // T * (H + 1)
  uint8_t* q_out;
  uint8_t* cache;
  int32_t* status;
};

// q / H for 0 <= q < 2^31 by one multiply-high: with M = ceil(2^64 / H),
// floor(q M / 2^64) = floor(q / H + q (M - 2^64/H) / 2^64), and the added term
// is below 2^-33 while the fractional part of q / H is at most 1 - 2^-16.
__device__ __forceinline__ int64_t div_heads(const Args& a, int64_t q) {
  return a.H == 1 ? q : static_cast<int64_t>(__umul64hi(static_cast<uint64_t>(q), a.h_magic));
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

// The divisor of an e4m3 output (scale read from device memory), or a dummy
// one that selects the branch-free path when the output is bf16.
template <bool FP8>
__device__ __forceinline__ Divisor divisor_of(const float* scale) {
  Divisor d{};
  d.fast = true;
  if constexpr (FP8) d = make_divisor(__ldg(scale));
  return d;
}

// ---- pieces of one row: a 16-byte nope chunk (8 values) and the RoPE pairs
// (i, i + 32), one pair (store_pe) or two adjacent pairs (store_pe2) at a
// time; the kernels decide which lane takes which piece.  Loads of data the
// upstream kernel may still be writing under programmatic dependent launch go
// to L2 only (.cg), never through the read-only path.

// Rotation of pair `i` for token t: (cos, sin) from the table row of its
// position, or `on` false when the position is out of range.
struct Rot {
  float c, s;
  bool on;
};

__device__ __forceinline__ Rot load_rotation(const Args& a, int64_t t, int i) {
  Rot r{1.0f, 0.0f, false};
  const int64_t pos = __ldg(a.positions + t);
  if (pos >= 0 && pos < a.rope_rows) {
    const float* row = a.cos_sin + pos * kPe;
    r.c = __ldg(row + i);
    r.s = __ldg(row + kHalfPe + i);
    r.on = true;
  }
  return r;
}

template <bool FP8, bool FAST>
__device__ __forceinline__ void store_nope(uint8_t* dst, int chunk, const uint4 v, const Divisor& d) {
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(dst + chunk * 8) = chunk_to_e4m3<FAST>(v, d);
  } else {
    *reinterpret_cast<uint4*>(dst + chunk * 16) = v;
  }
}

// RoPE pair i of a row: pe[i] in the low half of `pe`, pe[i+32] in the high half.
template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void store_pe(uint8_t* dst, int i, uint32_t pe, const Rot& r, const Divisor& d) {
  float a = bf16_lo(pe);
  float b = bf16_hi(pe);
  bool rotated = false;
  if constexpr (ROPE) {
    if (r.on) {
      float ya, yb;
      rope_pair(a, b, r.c, r.s, ya, yb);
      a = ya;
      b = yb;
      rotated = true;
    }
  }
  if constexpr (FP8) {
    const uint32_t p = e4m3x2_of_f32<FAST>(a, b, d);
    dst[kNope + i] = static_cast<uint8_t>(p & 0xffu);
    dst[kNope + kHalfPe + i] = static_cast<uint8_t>((p >> 8) & 0xffu);
  } else {
    const uint32_t p = rotated ? pack_bf16x2(a, b) : pe;  // unrotated: the input bits
    uint16_t* o = reinterpret_cast<uint16_t*>(dst);
    o[kNope + i] = static_cast<uint16_t>(p & 0xffffu);
    o[kNope + kHalfPe + i] = static_cast<uint16_t>(p >> 16);
  }
}

// RoPE pairs i0 and i0 + 1 of a row together (i0 even): a01 holds pe[i0],
// pe[i0+1] and b01 holds pe[i0+32], pe[i0+33]; the outputs go out as one
// 2-byte (e4m3) or 4-byte (bf16) store per half.  r0 and r1 rotate pairs i0
// and i0 + 1 (both on or both off: one position per token).
template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void store_pe2(uint8_t* dst, int i0, uint32_t a01, uint32_t b01, const Rot& r0,
                                          const Rot& r1, const Divisor& d) {
  bool rotated = false;
  float a0 = 0.0f, a1 = 0.0f, b0 = 0.0f, b1 = 0.0f;
  if constexpr (ROPE) {
    if (r0.on) {
      rope_pair(bf16_lo(a01), bf16_lo(b01), r0.c, r0.s, a0, b0);
      rope_pair(bf16_hi(a01), bf16_hi(b01), r1.c, r1.s, a1, b1);
      rotated = true;
    }
  }
  if constexpr (FP8) {
    uint32_t ea, eb;
    if (rotated) {
      ea = e4m3x2_of_f32<FAST>(a0, a1, d);
      eb = e4m3x2_of_f32<FAST>(b0, b1, d);
    } else {  // unrotated values are bf16: the quotient of bf16 inputs
      ea = e4m3x2_of_bf16x2<FAST>(a01, d);
      eb = e4m3x2_of_bf16x2<FAST>(b01, d);
    }
    *reinterpret_cast<uint16_t*>(dst + kNope + i0) = static_cast<uint16_t>(ea);
    *reinterpret_cast<uint16_t*>(dst + kNope + kHalfPe + i0) = static_cast<uint16_t>(eb);
  } else {
    *reinterpret_cast<uint32_t*>(dst + 2 * (kNope + i0)) = rotated ? pack_bf16x2(a0, a1) : a01;
    *reinterpret_cast<uint32_t*>(dst + 2 * (kNope + kHalfPe + i0)) = rotated ? pack_bf16x2(b0, b1) : b01;
  }
}

__device__ __forceinline__ uint4 ld_chunk(const uint16_t* row, int chunk) {
  return __ldcg(reinterpret_cast<const uint4*>(row) + chunk);
}

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* pe, int i) {
  return static_cast<uint32_t>(__ldcg(pe + i)) | (static_cast<uint32_t>(__ldcg(pe + kHalfPe + i)) << 16);
}

}  // namespace mla
