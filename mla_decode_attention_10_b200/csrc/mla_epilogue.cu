// mla_epilogue.cu -- the fused MLA decode epilogue for B200 (sm_100a) and its C-ABI launcher.
//
// Per token t: H latent query rows q_out[t, h] = enc(rope(q_nope[t, h] || q_pe[t, h]))
// and one latent cache row cache[slot_mapping[t]] = enc(rope(kv_c[t] || k_pe[t])),
// each 576 = 512 + 64 wide (vLLM PR #54896 report, 实现拆解 items 1-3 and the
// fusedKimiK3MLADecodeQConcatKVCacheKernel / writeLatent576 listing).
//
// The op moves bytes and does almost no arithmetic, so it is bound by HBM
// bandwidth at large T and by launch and memory latency at decode sizes; there
// is no contraction and no tensor-core work.  Two kernels share the element
// code (latent_math.cuh):
//
//   split kernel (small T): each row gets three warps, as the page's SPLIT=3
//     path does.  Warps 0 and 1 copy/convert the 64 nope chunks (16 bytes, 8
//     values, one chunk per lane); warp 2 does the 64 pe values as 32 RoPE
//     pairs (i, i+32), one pair per lane, so the rotation needs no shuffles.
//     Every lane issues its loads at once: the critical path is one
//     dependent load (position -> table row) plus the data load.
//   rows kernel (large T): one warp per row (lane: nope chunks lane and
//     lane+32, pe pair lane); the grid is a multiple of the SM count sized to
//     the resident blocks, each warp walks a contiguous range of rows, keeps
//     the next row's loads in flight while it converts the current one, and
//     looks up a token's rotation once for all of its adjacent rows.
//
// Row order: rows [0, T) are the T cache rows, rows [T, T + T*H) the query
// rows in q_out order.  Cache rows never wait on the upstream kernel, so
// under programmatic dependent launch they run while it finishes
// (PR #54896 report, 实现拆解 item 2); query rows execute griddepcontrol.wait
// right before they read q_nope / q_pe, after their slot, position, table and
// scale loads.  Every thread issues griddepcontrol.launch_dependents after its
// last store (the report's 评论区精华: the early trigger was a race).

#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "latent_math.cuh"
#include "mla_epilogue.h"

namespace mla {

constexpr int kNope = 512;
constexpr int kPe = 64;
constexpr int kHalfPe = 32;
constexpr int kRow = 576;
constexpr int kSplitThreadsPerRow = 96;
constexpr int kSplitMaxRowsPerBlock = 4;  // 384 threads
// Resident 256-thread blocks per SM the rows kernel is compiled for: 5 (a
// 48-register cap) for bf16 outputs; 6 (40 registers) when an output is
// e4m3, whose arithmetic leaves the kernel short of memory parallelism at 5
// (measured on B200: 0.75 -> 0.78 of copy bandwidth for T=8192, H=16; the
// bf16 variants lose at 6).
constexpr int kRowsMaxBlocksPerSm = 6;
constexpr int rows_blocks_per_sm(bool qf8, bool kvf8) { return (qf8 || kvf8) ? 6 : 5; }

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

// Rotation of pair `i` for token t: (cos, sin) from the table row of its position.
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

// Nope chunk `chunk` (8 values) of a row: 16 bytes in, 16 (bf16) or 8 (e4m3) out.
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

__device__ __forceinline__ uint4 ld_chunk(const uint16_t* row, int chunk) {
  return __ldcg(reinterpret_cast<const uint4*>(row) + chunk);
}

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* pe, int i) {
  return static_cast<uint32_t>(__ldcg(pe + i)) | (static_cast<uint32_t>(__ldcg(pe + kHalfPe + i)) << 16);
}

// ------------------------------------------------------------------------------------
// split kernel: three warps per row
// ------------------------------------------------------------------------------------

template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void split_query_row(const Args& a, int64_t q, int part, int lane, const Divisor& d) {
  const int64_t t = div_heads(a, q);
  const int64_t h = q - t * a.H;
  uint8_t* dst = a.q_out + q * (FP8 ? kRow : 2 * kRow);
  if (part < 2) {
    const uint16_t* src = a.q_nope + t * a.qn_st + h * a.qn_sh;
    const int chunk = part * 32 + lane;
    pdl_wait();
    const uint4 v = ld_chunk(src, chunk);
    store_nope<FP8, FAST>(dst, chunk, v, d);
  } else {
    const uint16_t* src = a.q_pe + t * a.qp_st + h * a.qp_sh;
    Rot r{1.0f, 0.0f, false};
    if constexpr (ROPE) r = load_rotation(a, t, lane);
    pdl_wait();
    const uint32_t pe = ld_pair(src, lane);
    store_pe<FP8, ROPE, FAST>(dst, lane, pe, r, d);
  }
}

template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void split_cache_row(const Args& a, int64_t t, int part, int lane, const Divisor& d) {
  const int64_t slot = __ldg(a.slots + t);
  const bool in_range = slot >= 0 && slot < a.cache_rows;
  uint8_t* dst = a.cache + (in_range ? slot : 0) * (FP8 ? kRow : 2 * kRow);
  if (part < 2) {
    const int chunk = part * 32 + lane;
    const uint4 v = ld_chunk(a.kv_c + t * a.kv_st, chunk);
    if (part == 0 && lane == 0 && slot >= a.cache_rows) report(a.status, MLA_STATUS_SLOT_RANGE);
    if (in_range) store_nope<FP8, FAST>(dst, chunk, v, d);
  } else {
    Rot r{1.0f, 0.0f, false};
    if constexpr (ROPE) {
      r = load_rotation(a, t, lane);
      if (lane == 0 && !r.on) report(a.status, MLA_STATUS_POS_RANGE);
    }
    const uint32_t pe = ld_pair(a.k_pe + t * a.kp_st, lane);
    if (in_range) store_pe<FP8, ROPE, FAST>(dst, lane, pe, r, d);
  }
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(kSplitThreadsPerRow * kSplitMaxRowsPerBlock) mla_epilogue_split_kernel(const Args a) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int rows_per_block = blockDim.x / kSplitThreadsPerRow;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * rows_per_block + warp / 3;
  const int part = warp % 3;
  if (g < a.rows) {
    // the row's divisor (scales are read before any wait); quotients take the
    // corrected-reciprocal path unless the scale is outside [2^-64, 2^64]
    if (g < a.T) {
      Divisor d{};
      d.fast = true;
      if constexpr (KVF8) d = make_divisor(__ldg(a.kv_scale));
      if (d.fast) {
        split_cache_row<KVF8, ROPE, true>(a, g, part, lane, d);
      } else {
        split_cache_row<KVF8, ROPE, false>(a, g, part, lane, d);
      }
    } else {
      Divisor d{};
      d.fast = true;
      if constexpr (QF8) d = make_divisor(__ldg(a.q_scale));
      if (d.fast) {
        split_query_row<QF8, ROPE, true>(a, g - a.T, part, lane, d);
      } else {
        split_query_row<QF8, ROPE, false>(a, g - a.T, part, lane, d);
      }
    }
  }
  pdl_trigger();
}

// ------------------------------------------------------------------------------------
// rows kernel: one warp per row, grid-stride over rows
// ------------------------------------------------------------------------------------

template <bool QF8, bool KVF8, bool ROPE, bool FAST>
__device__ __forceinline__ void rows_body(const Args& a, const Divisor& dq, const Divisor& dk) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t wid = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  bool waited = false;

  for (int64_t g = wid; g < a.rows; g += warps) {
    // 1. addresses, slot and rotation: nothing here depends on the upstream kernel
    const bool is_cache = g < a.T;
    int64_t t;
    const uint16_t* nope;
    const uint16_t* pe;
    uint8_t* dst = nullptr;
    if (is_cache) {
      t = g;
      nope = a.kv_c + t * a.kv_st;
      pe = a.k_pe + t * a.kp_st;
      const int64_t slot = __ldg(a.slots + t);
      if (slot >= 0 && slot < a.cache_rows) {
        dst = a.cache + slot * (KVF8 ? kRow : 2 * kRow);
      } else if (slot >= a.cache_rows && lane == 0) {
        report(a.status, MLA_STATUS_SLOT_RANGE);
      }
    } else {
      const int64_t q = g - a.T;
      t = div_heads(a, q);
      const int64_t h = q - t * a.H;
      nope = a.q_nope + t * a.qn_st + h * a.qn_sh;
      pe = a.q_pe + t * a.qp_st + h * a.qp_sh;
      dst = a.q_out + q * (QF8 ? kRow : 2 * kRow);
    }
    Rot rot{1.0f, 0.0f, false};
    if constexpr (ROPE) {
      rot = load_rotation(a, t, lane);
      if (is_cache && lane == 0 && !rot.on) report(a.status, MLA_STATUS_POS_RANGE);
    }

    // 2. query rows read what the upstream kernel wrote: wait for it once
    if (!is_cache && !waited) {
      pdl_wait();
      waited = true;
    }

    // 3. the row's loads, then 4. convert and store
    const uint4 n0 = ld_chunk(nope, lane);
    const uint4 n1 = ld_chunk(nope, lane + 32);
    const uint32_t p = ld_pair(pe, lane);
    if (dst == nullptr) continue;
    if (is_cache) {
      store_nope<KVF8, FAST>(dst, lane, n0, dk);
      store_nope<KVF8, FAST>(dst, lane + 32, n1, dk);
      store_pe<KVF8, ROPE, FAST>(dst, lane, p, rot, dk);
    } else {
      store_nope<QF8, FAST>(dst, lane, n0, dq);
      store_nope<QF8, FAST>(dst, lane + 32, n1, dq);
      store_pe<QF8, ROPE, FAST>(dst, lane, p, rot, dq);
    }
  }
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(256, rows_blocks_per_sm(QF8, KVF8)) mla_epilogue_rows_kernel(const Args a) {
  // scales are read before any wait; the whole body takes the corrected-
  // reciprocal quotient unless a scale is outside [2^-64, 2^64]
  Divisor dq{}, dk{};
  dq.fast = dk.fast = true;
  if constexpr (QF8) dq = make_divisor(__ldg(a.q_scale));
  if constexpr (KVF8) dk = make_divisor(__ldg(a.kv_scale));
  if (dq.fast && dk.fast) {
    rows_body<QF8, KVF8, ROPE, true>(a, dq, dk);
  } else {
    rows_body<QF8, KVF8, ROPE, false>(a, dq, dk);
  }
  pdl_trigger();
}

// kernel tables indexed by (ROPE, Q_FP8, KV_FP8) = flags & 7
template <int F>
const void* split_kernel_for() {
  return reinterpret_cast<const void*>(
      &mla_epilogue_split_kernel<(F & MLA_FLAG_Q_FP8) != 0, (F & MLA_FLAG_KV_FP8) != 0, (F & MLA_FLAG_ROPE) != 0>);
}
template <int F>
const void* rows_kernel_for() {
  return reinterpret_cast<const void*>(
      &mla_epilogue_rows_kernel<(F & MLA_FLAG_Q_FP8) != 0, (F & MLA_FLAG_KV_FP8) != 0, (F & MLA_FLAG_ROPE) != 0>);
}

const void* const kSplitKernels[8] = {split_kernel_for<0>(), split_kernel_for<1>(), split_kernel_for<2>(),
                                      split_kernel_for<3>(), split_kernel_for<4>(), split_kernel_for<5>(),
                                      split_kernel_for<6>(), split_kernel_for<7>()};
const void* const kRowsKernels[8] = {rows_kernel_for<0>(), rows_kernel_for<1>(), rows_kernel_for<2>(),
                                     rows_kernel_for<3>(), rows_kernel_for<4>(), rows_kernel_for<5>(),
                                     rows_kernel_for<6>(), rows_kernel_for<7>()};

}  // namespace mla

// ======================================================================================
// host side: validation, plan, launch
// ======================================================================================

namespace {

constexpr uint32_t kKnownFlags = MLA_FLAG_ROPE | MLA_FLAG_Q_FP8 | MLA_FLAG_KV_FP8 | MLA_FLAG_PDL |
                                 MLA_FLAG_FORCE_SPLIT | MLA_FLAG_FORCE_ROWS;
constexpr int kMaxDevices = 64;

mla_tuning g_tuning = {4608, 2, 8, mla::kRowsMaxBlocksPerSm};
int g_sm_count[kMaxDevices] = {0};
thread_local int32_t g_last_cuda_error = 0;

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

mla_status device_sm_count(int32_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices)) e = cudaErrorInvalidDevice;
  if (e == cudaSuccess && g_sm_count[dev] <= 0) {
    int n = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) g_sm_count[dev] = n;
  }
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int32_t>(e);
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  *out = g_sm_count[dev];
  return MLA_OK;
}

mla_status make_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* p) {
  const int64_t rows = T * (H + 1);
  const bool split = (flags & MLA_FLAG_FORCE_SPLIT) ? true
                     : (flags & MLA_FLAG_FORCE_ROWS) ? false
                                                      : (rows <= g_tuning.split_max_rows);
  p->sm_count = sm_count;
  if (split) {
    const int32_t rpb = g_tuning.split_rows_per_block;
    p->mode = MLA_MODE_SPLIT;
    p->rows_per_block = rpb;
    p->threads_per_block = mla::kSplitThreadsPerRow * rpb;
    p->blocks = (rows + rpb - 1) / rpb;
  } else {
    const int32_t w = g_tuning.rows_warps_per_block;
    const int64_t per_block = w;
    const int64_t need = (rows + per_block - 1) / per_block;
    const int32_t resident = mla::rows_blocks_per_sm((flags & MLA_FLAG_Q_FP8) != 0, (flags & MLA_FLAG_KV_FP8) != 0);
    const int32_t per_sm = g_tuning.rows_blocks_per_sm < resident ? g_tuning.rows_blocks_per_sm : resident;
    const int64_t cap = static_cast<int64_t>(sm_count) * per_sm;
    p->mode = MLA_MODE_ROWS;
    p->rows_per_block = 1;
    p->threads_per_block = 32 * w;
    p->blocks = need < cap ? need : cap;
  }
  return MLA_OK;
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG: null pointer, bad size or stride, or conflicting flags";
    case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT: a pointer or stride breaks the 16-byte row rule";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED: unknown flag bit";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: the CUDA runtime refused the launch";
  }
  return "unknown mla_status";
}

int32_t mla_last_cuda_error(void) { return g_last_cuda_error; }

void mla_epilogue_set_tuning(const mla_tuning* t) {
  if (t == nullptr) return;
  if (t->split_max_rows > 0) g_tuning.split_max_rows = t->split_max_rows;
  if (t->split_rows_per_block > 0)
    g_tuning.split_rows_per_block = t->split_rows_per_block < mla::kSplitMaxRowsPerBlock ? t->split_rows_per_block
                                                                                          : mla::kSplitMaxRowsPerBlock;
  if (t->rows_warps_per_block > 0) g_tuning.rows_warps_per_block = t->rows_warps_per_block < 8 ? t->rows_warps_per_block : 8;
  if (t->rows_blocks_per_sm > 0)
    g_tuning.rows_blocks_per_sm =
        t->rows_blocks_per_sm < mla::kRowsMaxBlocksPerSm ? t->rows_blocks_per_sm : mla::kRowsMaxBlocksPerSm;
}

void mla_epilogue_get_tuning(mla_tuning* out) {
  if (out != nullptr) *out = g_tuning;
}

mla_status mla_epilogue_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* out) {
  if (out == nullptr || T < 1 || H < 1 || H > 65536) return MLA_ERR_INVALID_ARG;
  if ((flags & MLA_FLAG_FORCE_SPLIT) && (flags & MLA_FLAG_FORCE_ROWS)) return MLA_ERR_INVALID_ARG;
  if (T > (static_cast<int64_t>(INT_MAX)) / (H + 1)) return MLA_ERR_INVALID_ARG;
  if (sm_count <= 0) {
    const mla_status s = device_sm_count(&sm_count);
    if (s != MLA_OK) return s;
  }
  return make_plan(T, H, flags, sm_count, out);
}

mla_status mla_epilogue_launch(
    const void* q_nope, int64_t q_nope_stride_t, int64_t q_nope_stride_h,
    const void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
    const void* kv_c, int64_t kv_c_stride_t,
    const void* k_pe, int64_t k_pe_stride_t,
    const int64_t* slot_mapping, const int32_t* positions,
    const float* cos_sin, int64_t rope_rows,
    const float* q_scale, const float* kv_scale,
    int64_t T, int64_t H, int64_t block_size, int64_t num_blocks,
    uint32_t flags, void* q_out, void* cache, int32_t* status, mla_stream_t stream) {
  // ---- scalars and flags
  if ((flags & ~kKnownFlags) != 0) return MLA_ERR_UNSUPPORTED;
  if ((flags & MLA_FLAG_FORCE_SPLIT) && (flags & MLA_FLAG_FORCE_ROWS)) return MLA_ERR_INVALID_ARG;
  if (T < 0 || H < 1 || H > 65536 || block_size < 1 || num_blocks < 0) return MLA_ERR_INVALID_ARG;
  if (T > static_cast<int64_t>(INT_MAX) / (H + 1)) return MLA_ERR_INVALID_ARG;
  if (num_blocks > (INT64_C(1) << 50) / block_size) return MLA_ERR_INVALID_ARG;
  const bool rope = (flags & MLA_FLAG_ROPE) != 0;
  const bool qf8 = (flags & MLA_FLAG_Q_FP8) != 0;
  const bool kvf8 = (flags & MLA_FLAG_KV_FP8) != 0;
  if (rope && (rope_rows < 1 || rope_rows > (INT64_C(1) << 40))) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  const int64_t cache_rows = num_blocks * block_size;

  // ---- pointers
  if (q_nope == nullptr || q_pe == nullptr || kv_c == nullptr || k_pe == nullptr || slot_mapping == nullptr ||
      q_out == nullptr || (cache == nullptr && cache_rows > 0))
    return MLA_ERR_INVALID_ARG;
  if (rope && (positions == nullptr || cos_sin == nullptr)) return MLA_ERR_INVALID_ARG;
  if ((qf8 && q_scale == nullptr) || (kvf8 && kv_scale == nullptr)) return MLA_ERR_INVALID_ARG;
  if (q_nope_stride_t < 0 || q_nope_stride_h < 0 || q_pe_stride_t < 0 || q_pe_stride_h < 0 || kv_c_stride_t < 0 ||
      k_pe_stride_t < 0)
    return MLA_ERR_INVALID_ARG;

  // ---- alignment: 16-byte rows for the vectorised parts
  if (!aligned(q_nope, 16) || !aligned(kv_c, 16) || !aligned(q_out, 16) || (cache != nullptr && !aligned(cache, 16)))
    return MLA_ERR_ALIGNMENT;
  if ((T > 1 && (q_nope_stride_t % 8) != 0) || (H > 1 && (q_nope_stride_h % 8) != 0) ||
      (T > 1 && (kv_c_stride_t % 8) != 0))
    return MLA_ERR_ALIGNMENT;
  if (!aligned(q_pe, 2) || !aligned(k_pe, 2) || !aligned(slot_mapping, 8)) return MLA_ERR_ALIGNMENT;
  if ((rope && (!aligned(positions, 4) || !aligned(cos_sin, 4))) || (qf8 && !aligned(q_scale, 4)) ||
      (kvf8 && !aligned(kv_scale, 4)) || (status != nullptr && !aligned(status, 4)))
    return MLA_ERR_ALIGNMENT;

  // ---- plan and launch
  int32_t sms = 0;
  mla_status s = device_sm_count(&sms);
  if (s != MLA_OK) return s;
  mla_plan plan;
  s = make_plan(T, H, flags, sms, &plan);
  if (s != MLA_OK) return s;

  mla::Args a;
  a.q_nope = static_cast<const uint16_t*>(q_nope);
  a.qn_st = q_nope_stride_t;
  a.qn_sh = q_nope_stride_h;
  a.q_pe = static_cast<const uint16_t*>(q_pe);
  a.qp_st = q_pe_stride_t;
  a.qp_sh = q_pe_stride_h;
  a.kv_c = static_cast<const uint16_t*>(kv_c);
  a.kv_st = kv_c_stride_t;
  a.k_pe = static_cast<const uint16_t*>(k_pe);
  a.kp_st = k_pe_stride_t;
  a.slots = slot_mapping;
  a.positions = positions;
  a.cos_sin = cos_sin;
  a.rope_rows = rope ? rope_rows : 0;
  a.q_scale = q_scale;
  a.kv_scale = kv_scale;
  a.T = T;
  a.H = H;
  a.h_magic = H > 1 ? (UINT64_MAX / static_cast<uint64_t>(H)) + 1 : 0;
  a.cache_rows = cache_rows;
  a.rows = T * (H + 1);
  a.q_out = static_cast<uint8_t*>(q_out);
  a.cache = static_cast<uint8_t*>(cache);
  a.status = status;

  const int k = static_cast<int>(flags & 7u);
  const void* fn = (plan.mode == MLA_MODE_SPLIT) ? mla::kSplitKernels[k] : mla::kRowsKernels[k];

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.blocks), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(plan.threads_per_block), 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  if (flags & MLA_FLAG_PDL) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  void* args[] = {&a};
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) {
    g_last_cuda_error = static_cast<int32_t>(e);
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

}  // extern "C"
