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
  uint64_t h_magic;  // ceil(2^64 / H) for H >= 2, see div_heads
  int64_t cache_rows;
  int64_t rows;  // T * (H + 1)
  uint8_t* q_out;
  uint8_t* cache;
  int32_t* status;
  // 16-byte vector access is possible (base 16-byte aligned, strides
  // multiples of 8 elements): q_pe rows, k_pe rows, cos_sin rows
  int32_t qpe_vec, kpe_vec, tab_vec;
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

// Loads that read what the upstream kernel may still be writing under
// programmatic dependent launch: L2 only (.cg), never the read-only path.
__device__ __forceinline__ uint4 ld_cg16(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

}  // namespace mla
