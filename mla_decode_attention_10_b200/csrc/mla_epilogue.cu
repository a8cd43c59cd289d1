// mla_epilogue.cu -- the fused MLA decode epilogue for B200 (sm_100a): the
// small-batch kernels and the C-ABI launcher.
//
// Per token t: H latent query rows q_out[t, h] = enc(rope(q_nope[t, h] || q_pe[t, h]))
// and one latent cache row cache[slot_mapping[t]] = enc(rope(kv_c[t] || k_pe[t])),
// each 576 = 512 + 64 wide (vLLM PR #54896 report, 实现拆解 items 1-3 and the
// fusedKimiK3MLADecodeQConcatKVCacheKernel / writeLatent576 listing).
//
// The op moves bytes and does almost no arithmetic: at decode sizes it is
// bound by launch and memory latency, at large T by HBM bandwidth; there is
// no contraction and no tensor-core work.  Three launch modes:
//
//   SPLIT (small T): every row gets 68 threads.  64 of them move one 16-byte
//     nope chunk each (8 values); 4 of them each own the pe octets 8j..8j+7
//     and 32+8j..32+8j+7, so one thread holds both members of its 8 RoPE
//     pairs (i, i+32) and rotates them without shuffles, with 16-byte loads
//     and 16-byte (bf16) or 8-byte (e4m3) stores.  Threads map to work by
//     their index in the grid: the first 4 * rows threads are the pe threads
//     of all rows (eight rows per warp; their position -> table chain is the
//     longest, and blocks start in index order), the next 64 * rows the nope
//     threads, so every warp has one role and the block size is free.  At
//     decode sizes the latency is lowest when the work is spread over as
//     many SMs as there are (measured on B200: one 17-row token in 37
//     one-warp blocks is about 0.9 us faster than in one to three blocks),
//     so the plan sizes blocks to give about one block per SM; for T = 1
//     that is one-warp blocks (the num_tokens == 1 case of PR #53526,
//     关联脉络).
//   ROWS (large T): mla_rows.cu.
//
// In SPLIT every thread computes its addresses and loads its slot,
// position, table entries and scale before griddepcontrol.wait; after the
// wait a query-row thread has one load -> convert -> store left (PR #54896
// report, 实现拆解 item 2).  Cache rows never wait.  Every thread issues
// griddepcontrol.launch_dependents after its last store (the report's
// 评论区精华: the early trigger was a race).

#include <atomic>
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "epilogue_device.cuh"
#include "mla_epilogue.h"
#include "mla_rows.h"
#include "mla_runtime.h"

namespace mla {

constexpr int kSmallMaxThreads = 1024;
constexpr int kSmallThreadsPerRow = 68;  // 64 nope threads + 4 pe threads

// Nope chunk `chunk` (8 values) of a row: 16 bytes in, 16 (bf16) or 8 (e4m3) out.
template <bool FP8, bool FAST>
__device__ __forceinline__ void store_nope(uint8_t* dst, int chunk, const uint4 v, const Divisor& d) {
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(dst + chunk * 8) = chunk_to_e4m3<FAST>(v, d);
  } else {
    *reinterpret_cast<uint4*>(dst + chunk * 16) = v;
  }
}

// Rotation of the pairs 8j .. 8j+7 of token t: cos and sin from the table row
// of its position, or `on` false when RoPE is off or the position is out of
// range.
struct Rot8 {
  float c[8], s[8];
  bool on;
};

template <bool ROPE>
__device__ __forceinline__ Rot8 load_rot8(const Args& a, int64_t t, int j) {
  Rot8 r;
  r.on = false;
  if constexpr (ROPE) {
    const int64_t pos = __ldg(a.positions + t);
    if (pos >= 0 && pos < a.rope_rows) {
      const float* row = a.cos_sin + pos * kPe + 8 * j;
      if (a.tab_vec) {
        const float4 c0 = __ldg(reinterpret_cast<const float4*>(row));
        const float4 c1 = __ldg(reinterpret_cast<const float4*>(row) + 1);
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(row + kHalfPe));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(row + kHalfPe) + 1);
        r.c[0] = c0.x; r.c[1] = c0.y; r.c[2] = c0.z; r.c[3] = c0.w;
        r.c[4] = c1.x; r.c[5] = c1.y; r.c[6] = c1.z; r.c[7] = c1.w;
        r.s[0] = s0.x; r.s[1] = s0.y; r.s[2] = s0.z; r.s[3] = s0.w;
        r.s[4] = s1.x; r.s[5] = s1.y; r.s[6] = s1.z; r.s[7] = s1.w;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          r.c[k] = __ldg(row + k);
          r.s[k] = __ldg(row + kHalfPe + k);
        }
      }
      r.on = true;
    }
  }
  return r;
}

// pe values 8j .. 8j+7 (`lo`) and 32+8j .. 32+8j+7 (`hi`) of one row as bf16
// words (value 2k in the low half of word k): two 16-byte loads when the row
// is 16-byte aligned, else sixteen 2-byte loads.
__device__ __forceinline__ void load_pe8(const uint16_t* pe, int j, bool vec, uint4& lo, uint4& hi) {
  if (vec) {
    lo = ld_cg16(pe + 8 * j);
    hi = ld_cg16(pe + kHalfPe + 8 * j);
  } else {
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      w[k] = static_cast<uint32_t>(__ldcg(pe + 8 * j + 2 * k)) |
             (static_cast<uint32_t>(__ldcg(pe + 8 * j + 2 * k + 1)) << 16);
      w[4 + k] = static_cast<uint32_t>(__ldcg(pe + kHalfPe + 8 * j + 2 * k)) |
                 (static_cast<uint32_t>(__ldcg(pe + kHalfPe + 8 * j + 2 * k + 1)) << 16);
    }
    lo = make_uint4(w[0], w[1], w[2], w[3]);
    hi = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// The 8 RoPE pairs (8j + k, 32 + 8j + k), k < 8, of a row: rotate in fp32, encode,
// store 2 x 16 bytes (bf16) or 2 x 8 bytes (e4m3).
template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void store_pe8(uint8_t* row, int j, const uint4 lo, const uint4 hi, const Rot8& r,
                                          const Divisor& d) {
  const uint32_t wl[4] = {lo.x, lo.y, lo.z, lo.w};
  const uint32_t wh[4] = {hi.x, hi.y, hi.z, hi.w};
  float ya[8], yb[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float a = (k & 1) ? bf16_hi(wl[k >> 1]) : bf16_lo(wl[k >> 1]);
    const float b = (k & 1) ? bf16_hi(wh[k >> 1]) : bf16_lo(wh[k >> 1]);
    ya[k] = a;
    yb[k] = b;
    if (ROPE && r.on) rope_pair(a, b, r.c[k], r.s[k], ya[k], yb[k]);
  }
  if constexpr (FP8) {
    uint2 oa, ob;
    oa.x = e4m3x2_of_f32<FAST>(ya[0], ya[1], d) | (e4m3x2_of_f32<FAST>(ya[2], ya[3], d) << 16);
    oa.y = e4m3x2_of_f32<FAST>(ya[4], ya[5], d) | (e4m3x2_of_f32<FAST>(ya[6], ya[7], d) << 16);
    ob.x = e4m3x2_of_f32<FAST>(yb[0], yb[1], d) | (e4m3x2_of_f32<FAST>(yb[2], yb[3], d) << 16);
    ob.y = e4m3x2_of_f32<FAST>(yb[4], yb[5], d) | (e4m3x2_of_f32<FAST>(yb[6], yb[7], d) << 16);
    *reinterpret_cast<uint2*>(row + kNope + 8 * j) = oa;
    *reinterpret_cast<uint2*>(row + kNope + kHalfPe + 8 * j) = ob;
  } else {
    uint4 oa = lo, ob = hi;  // unrotated values keep their bits (NaN payloads included)
    if (ROPE && r.on) {
      oa = make_uint4(pack_bf16x2(ya[0], ya[1]), pack_bf16x2(ya[2], ya[3]), pack_bf16x2(ya[4], ya[5]),
                      pack_bf16x2(ya[6], ya[7]));
      ob = make_uint4(pack_bf16x2(yb[0], yb[1]), pack_bf16x2(yb[2], yb[3]), pack_bf16x2(yb[4], yb[5]),
                      pack_bf16x2(yb[6], yb[7]));
    }
    *reinterpret_cast<uint4*>(row + 2 * (kNope + 8 * j)) = oa;
    *reinterpret_cast<uint4*>(row + 2 * (kNope + kHalfPe + 8 * j)) = ob;
  }
}

// ------------------------------------------------------------------------------------
// small-batch kernel
// ------------------------------------------------------------------------------------

// A row's e4m3 scale: its load is issued with the row's other loads and the
// divisor is made only when the stores need it, so the scale adds no step
// to the row's chain of dependent loads.
template <bool FP8>
__device__ __forceinline__ float scale_of(const float* scale) {
  if constexpr (FP8) return __ldg(scale);
  return 1.0f;
}

template <bool FP8>
__device__ __forceinline__ Divisor divisor_from(float scale) {
  Divisor d{};
  d.fast = true;
  if constexpr (FP8) d = make_divisor(scale);
  return d;
}

// Stores of one thread's share of a row, the quotient path chosen from the
// scale: the corrected reciprocal unless the scale is outside [2^-64, 2^64].
template <bool FP8, bool ROPE>
__device__ __forceinline__ void store_part(uint8_t* dst, bool pe, int part, const uint4& v, const uint4& lo,
                                           const uint4& hi, const Rot8& rot, float scale) {
  const Divisor d = divisor_from<FP8>(scale);
  if (!FP8 || d.fast) {
    if (!pe) {
      store_nope<FP8, true>(dst, part, v, d);
    } else {
      store_pe8<FP8, ROPE, true>(dst, part, lo, hi, rot, d);
    }
  } else {
    if (!pe) {
      store_nope<FP8, false>(dst, part, v, d);
    } else {
      store_pe8<FP8, ROPE, false>(dst, part, lo, hi, rot, d);
    }
  }
}

template <bool FP8, bool ROPE>
__device__ __forceinline__ void small_cache_row(const Args& a, int64_t t, bool pe, int part) {
  const float scale = scale_of<FP8>(a.kv_scale);
  const int64_t slot = __ldg(a.slots + t);
  uint4 v = make_uint4(0, 0, 0, 0), lo = v, hi = v;
  Rot8 rot;
  rot.on = false;
  if (!pe) {
    v = ld_cg16(a.kv_c + t * a.kv_st + 8 * part);
  } else {
    rot = load_rot8<ROPE>(a, t, part);
    load_pe8(a.k_pe + t * a.kp_st, part, a.kpe_vec != 0, lo, hi);
  }
  const bool in_range = slot >= 0 && slot < a.cache_rows;
  if (part == 0) {
    if (!pe && slot >= a.cache_rows) report(a.status, MLA_STATUS_SLOT_RANGE);
    if (ROPE && pe && !rot.on) report(a.status, MLA_STATUS_POS_RANGE);
  }
  if (in_range) store_part<FP8, ROPE>(a.cache + slot * (FP8 ? kRow : 2 * kRow), pe, part, v, lo, hi, rot, scale);
}

template <bool FP8, bool ROPE>
__device__ __forceinline__ void small_query_row(const Args& a, int64_t q, bool pe, int part) {
  const float scale = scale_of<FP8>(a.q_scale);
  const int64_t t = div_heads(a, q);
  const int64_t h = q - t * a.H;
  uint4 v = make_uint4(0, 0, 0, 0), lo = v, hi = v;
  Rot8 rot;
  rot.on = false;
  if (!pe) {
    const uint16_t* src = a.q_nope + t * a.qn_st + h * a.qn_sh + 8 * part;
    pdl_wait();
    v = ld_cg16(src);
  } else {
    const uint16_t* src = a.q_pe + t * a.qp_st + h * a.qp_sh;
    rot = load_rot8<ROPE>(a, t, part);
    pdl_wait();
    load_pe8(src, part, a.qpe_vec != 0, lo, hi);
  }
  store_part<FP8, ROPE>(a.q_out + q * (FP8 ? kRow : 2 * kRow), pe, part, v, lo, hi, rot, scale);
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(kSmallMaxThreads) mla_epilogue_small_kernel(const Args a) {
  // thread -> (row, part) by its index in the grid: the pe threads of all
  // rows first (4 per row: their position -> table chain is the longest, and
  // blocks are dispatched in index order), then the nope threads (64 per row)
  const int64_t gt = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t pe_threads = 4 * a.rows;
  const bool pe = gt < pe_threads;
  const int64_t u = pe ? gt : gt - pe_threads;
  const int64_t g = pe ? (u >> 2) : (u >> 6);
  const int part = static_cast<int>(pe ? (u & 3) : (u & 63));
  if (g < a.rows) {
    if (g < a.T) {
      small_cache_row<KVF8, ROPE>(a, g, pe, part);
    } else {
      small_query_row<QF8, ROPE>(a, g - a.T, pe, part);
    }
  }
  pdl_trigger();
}

// kernel tables indexed by (ROPE, Q_FP8, KV_FP8) = flags & 7
template <int F>
const void* small_kernel_for() {
  return reinterpret_cast<const void*>(
      &mla_epilogue_small_kernel<(F & MLA_FLAG_Q_FP8) != 0, (F & MLA_FLAG_KV_FP8) != 0, (F & MLA_FLAG_ROPE) != 0>);
}

const void* const kSplitKernels[8] = {small_kernel_for<0>(), small_kernel_for<1>(), small_kernel_for<2>(),
                                      small_kernel_for<3>(), small_kernel_for<4>(), small_kernel_for<5>(),
                                      small_kernel_for<6>(), small_kernel_for<7>()};

// ------------------------------------------------------------------------------------
// host helpers shared by every launcher (mla_runtime.h)
// ------------------------------------------------------------------------------------

namespace {
thread_local int32_t g_last_cuda_error = 0;
std::atomic<int32_t> g_sm_count[kMaxDevices];
}  // namespace

mla_status cuda_failure(cudaError_t e) {
  g_last_cuda_error = static_cast<int32_t>(e);
  (void)cudaGetLastError();
  return MLA_ERR_CUDA;
}

mla_status current_device(int* dev_out, int32_t* sm_count) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices)) e = cudaErrorInvalidDevice;
  if (e != cudaSuccess) return cuda_failure(e);
  int32_t n = g_sm_count[dev].load(std::memory_order_relaxed);
  if (n <= 0) {
    int v = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_failure(e);
    n = v;
    g_sm_count[dev].store(n, std::memory_order_relaxed);
  }
  if (dev_out != nullptr) *dev_out = dev;
  *sm_count = n;
  return MLA_OK;
}

}  // namespace mla

// ======================================================================================
// host side: validation, plan, launch
// ======================================================================================

namespace {

constexpr uint32_t kKnownFlags = MLA_FLAG_ROPE | MLA_FLAG_Q_FP8 | MLA_FLAG_KV_FP8 | MLA_FLAG_PDL |
                                 MLA_FLAG_FORCE_SPLIT | MLA_FLAG_FORCE_ROWS;

mla_tuning g_tuning = {4608, 0, mla::kRowsDefaultWarps, mla::kRowsMaxBlocksPerSm};

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

bool one_force_flag(uint32_t flags) {
  return !((flags & MLA_FLAG_FORCE_SPLIT) && (flags & MLA_FLAG_FORCE_ROWS));
}

// Threads per SPLIT block: the tuning value, or (0) the smallest multiple of
// 32 that gives at most one block per SM, between 32 and 1024.
int32_t split_threads(int64_t rows, int32_t sm_count) {
  if (g_tuning.split_threads_per_block > 0) return g_tuning.split_threads_per_block;
  const int64_t threads = mla::kSmallThreadsPerRow * rows;
  int64_t per = (threads + sm_count - 1) / sm_count;
  per = (per + 31) / 32 * 32;
  return static_cast<int32_t>(per < 32 ? 32 : (per > mla::kSmallMaxThreads ? mla::kSmallMaxThreads : per));
}

mla_status make_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* p) {
  const int64_t rows = T * (H + 1);
  const bool split = (flags & MLA_FLAG_FORCE_SPLIT)  ? true
                     : (flags & MLA_FLAG_FORCE_ROWS) ? false
                                                      : rows <= g_tuning.split_max_rows;
  p->sm_count = sm_count;
  if (split) {
    const int32_t tpb = split_threads(rows, sm_count);
    p->mode = MLA_MODE_SPLIT;
    p->rows_per_block = 0;
    p->threads_per_block = tpb;
    p->blocks = (mla::kSmallThreadsPerRow * rows + tpb - 1) / tpb;
    if (p->blocks > INT_MAX) {  // a small tuned block size on a huge forced launch
      p->threads_per_block = mla::kSmallMaxThreads;
      p->blocks = (mla::kSmallThreadsPerRow * rows + mla::kSmallMaxThreads - 1) / mla::kSmallMaxThreads;
    }
  } else {
    mla::rows_plan(rows, (flags & MLA_FLAG_Q_FP8) != 0, (flags & MLA_FLAG_KV_FP8) != 0, sm_count,
                   g_tuning.rows_blocks_per_sm, g_tuning.rows_warps_per_block, p);
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
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA: the CUDA runtime refused the call";
  }
  return "unknown mla_status";
}

int32_t mla_last_cuda_error(void) { return mla::g_last_cuda_error; }

void mla_epilogue_set_tuning(const mla_tuning* t) {
  if (t == nullptr) return;
  if (t->split_max_rows > 0) g_tuning.split_max_rows = t->split_max_rows;
  if (t->split_threads_per_block > 0) {
    const int32_t v = (t->split_threads_per_block + 31) / 32 * 32;
    g_tuning.split_threads_per_block = v < mla::kSmallMaxThreads ? v : mla::kSmallMaxThreads;
  } else if (t->split_threads_per_block < 0) {
    g_tuning.split_threads_per_block = 0;  // back to the automatic block size
  }
  if (t->rows_warps_per_block > 0)
    g_tuning.rows_warps_per_block =
        t->rows_warps_per_block < mla::kRowsMaxWarps ? t->rows_warps_per_block : mla::kRowsMaxWarps;
  if (t->rows_blocks_per_sm > 0)
    g_tuning.rows_blocks_per_sm =
        t->rows_blocks_per_sm < mla::kRowsMaxBlocksPerSm ? t->rows_blocks_per_sm : mla::kRowsMaxBlocksPerSm;
}

void mla_epilogue_get_tuning(mla_tuning* out) {
  if (out != nullptr) *out = g_tuning;
}

mla_status mla_epilogue_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* out) {
  if (out == nullptr || T < 1 || H < 1 || H > 65536) return MLA_ERR_INVALID_ARG;
  if (!one_force_flag(flags)) return MLA_ERR_INVALID_ARG;
  if (T > (static_cast<int64_t>(INT_MAX)) / (H + 1)) return MLA_ERR_INVALID_ARG;
  if (sm_count <= 0) {
    const mla_status s = mla::current_device(nullptr, &sm_count);
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
  if (!one_force_flag(flags)) return MLA_ERR_INVALID_ARG;
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
  mla_status s = mla::current_device(nullptr, &sms);
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
  a.qpe_vec = aligned(q_pe, 16) && (T == 1 || q_pe_stride_t % 8 == 0) && (H == 1 || q_pe_stride_h % 8 == 0);
  a.kpe_vec = aligned(k_pe, 16) && (T == 1 || k_pe_stride_t % 8 == 0);
  a.tab_vec = rope && aligned(cos_sin, 16);

  const int k = static_cast<int>(flags & 7u);
  const void* fn = nullptr;
  size_t smem = 0;
  if (plan.mode == MLA_MODE_SPLIT) {
    fn = mla::kSplitKernels[k];
  } else {
    s = mla::rows_kernel(k, plan.threads_per_block / 32, &fn, &smem);
    if (s != MLA_OK) return s;
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.blocks), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(plan.threads_per_block), 1, 1);
  cfg.dynamicSmemBytes = smem;
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
  if (e != cudaSuccess) return mla::cuda_failure(e);
  return MLA_OK;
}

}  // extern "C"
