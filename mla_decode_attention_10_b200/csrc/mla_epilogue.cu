// mla_epilogue.cu -- the fused MLA decode epilogue for B200 (sm_100a): the
// small-batch kernel and the C-ABI launcher.
//
// Per token t: H latent query rows q_out[t, h] = enc(rope(q_nope[t, h] || q_pe[t, h]))
// and one latent cache row cache[slot_mapping[t]] = enc(rope(kv_c[t] || k_pe[t])),
// each 576 = 512 + 64 wide (vLLM PR #54896 report, 实现拆解 items 1-3 and the
// fusedKimiK3MLADecodeQConcatKVCacheKernel / writeLatent576 listing).
//
// The op moves bytes and does almost no arithmetic: at decode sizes it is
// bound by launch and memory latency, at large T by HBM bandwidth; there is
// no contraction and no tensor-core work.  Two launch modes:
//
//   SPLIT (small T): every row gets three warps, as the page's SPLIT=3 path
//     does.  Warps 0 and 1 move the 64 nope chunks (16 bytes, 8 values, one
//     chunk per lane); warp 2 rotates the 64 pe values as 32 RoPE pairs
//     (i, i+32), one pair per lane, so the rotation needs no shuffles and
//     each thread's chain of dependent work stays short.  A block holds R
//     rows; at decode sizes latency falls as the rows spread over more SMs
//     (measured on B200), so the plan takes R = ceil(rows / SMs), at most 4:
//     one row per block for a single token (the num_tokens == 1 case of
//     PR #53526, 关联脉络), more rows per block only once every SM has one.
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

constexpr int kSplitThreadsPerRow = 96;  // three warps
constexpr int kSplitMaxRowsPerBlock = 10;  // 960 threads
constexpr int kSplitAutoMaxRows = 4;       // the automatic choice stops at 4 rows (measured best at T = 64 .. 256)

// A row's e4m3 scale: its load is issued with the row's other loads and the
// divisor is made only when the stores need it, so the scale adds no step
// to the row's chain of dependent loads.
template <bool FP8>
__device__ __forceinline__ float scale_of(const float* scale) {
  if constexpr (FP8) return __ldg(scale);
  return 1.0f;
}

// The stores of one lane's slice of a row (nope chunk `chunk` for parts 0
// and 1, pe pair `lane` for part 2), on the quotient path the scale selects:
// the corrected reciprocal unless the scale is outside [2^-64, 2^64].
template <bool FP8, bool ROPE>
__device__ __forceinline__ void split_store(uint8_t* dst, int part, int lane, const uint4& v, uint32_t pe,
                                            const Rot& rot, float scale) {
  Divisor d{};
  d.fast = true;
  if constexpr (FP8) d = make_divisor(scale);
  if (!FP8 || d.fast) {
    if (part < 2) {
      store_nope<FP8, true>(dst, part * 32 + lane, v, d);
    } else {
      store_pe<FP8, ROPE, true>(dst, lane, pe, rot, d);
    }
  } else {
    if (part < 2) {
      store_nope<FP8, false>(dst, part * 32 + lane, v, d);
    } else {
      store_pe<FP8, ROPE, false>(dst, lane, pe, rot, d);
    }
  }
}

template <bool FP8, bool ROPE>
__device__ __forceinline__ void split_cache_row(const Args& a, int64_t t, int part, int lane) {
  const float scale = scale_of<FP8>(a.kv_scale);
  const int64_t slot = __ldg(a.slots + t);
  uint4 v = make_uint4(0, 0, 0, 0);
  uint32_t pe = 0;
  Rot rot{1.0f, 0.0f, false};
  if (part < 2) {
    v = ld_chunk(a.kv_c + t * a.kv_st, part * 32 + lane);
  } else {
    pe = ld_pair(a.k_pe + t * a.kp_st, lane);
    if constexpr (ROPE) rot = load_rotation(a, t, lane);
  }
  if (lane == 0) {
    if (part == 0 && slot >= a.cache_rows) report(a.status, MLA_STATUS_SLOT_RANGE);
    if (ROPE && part == 2 && !rot.on) report(a.status, MLA_STATUS_POS_RANGE);
  }
  if (slot >= 0 && slot < a.cache_rows)
    split_store<FP8, ROPE>(a.cache + slot * (FP8 ? kRow : 2 * kRow), part, lane, v, pe, rot, scale);
}

template <bool FP8, bool ROPE>
__device__ __forceinline__ void split_query_row(const Args& a, int64_t q, int part, int lane) {
  const float scale = scale_of<FP8>(a.q_scale);
  const int64_t t = div_heads(a, q);
  const int64_t h = q - t * a.H;
  uint4 v = make_uint4(0, 0, 0, 0);
  uint32_t pe = 0;
  Rot rot{1.0f, 0.0f, false};
  if (part < 2) {
    const uint16_t* src = a.q_nope + t * a.qn_st + h * a.qn_sh;
    pdl_wait();
    v = ld_chunk(src, part * 32 + lane);
  } else {
    const uint16_t* src = a.q_pe + t * a.qp_st + h * a.qp_sh;
    if constexpr (ROPE) rot = load_rotation(a, t, lane);
    pdl_wait();
    pe = ld_pair(src, lane);
  }
  split_store<FP8, ROPE>(a.q_out + q * (FP8 ? kRow : 2 * kRow), part, lane, v, pe, rot, scale);
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(kSplitThreadsPerRow * kSplitMaxRowsPerBlock) mla_epilogue_split_kernel(const Args a) {
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int warp = static_cast<int>(threadIdx.x) >> 5;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x / kSplitThreadsPerRow) + warp / 3;
  const int part = warp % 3;
  if (g < a.rows) {
    if (g < a.T) {
      split_cache_row<KVF8, ROPE>(a, g, part, lane);
    } else {
      split_query_row<QF8, ROPE>(a, g - a.T, part, lane);
    }
  }
  pdl_trigger();
}

// kernel table indexed by (ROPE, Q_FP8, KV_FP8) = flags & 7
template <int F>
const void* split_kernel_for() {
  return reinterpret_cast<const void*>(
      &mla_epilogue_split_kernel<(F & MLA_FLAG_Q_FP8) != 0, (F & MLA_FLAG_KV_FP8) != 0, (F & MLA_FLAG_ROPE) != 0>);
}

const void* const kSplitKernels[8] = {split_kernel_for<0>(), split_kernel_for<1>(), split_kernel_for<2>(),
                                      split_kernel_for<3>(), split_kernel_for<4>(), split_kernel_for<5>(),
                                      split_kernel_for<6>(), split_kernel_for<7>()};

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

// Rows per SPLIT block: the tuning value, or (0) ceil(rows / SMs) up to 4,
// so that every SM gets a block before any block gets a second row.
int32_t split_rows(int64_t rows, int32_t sm_count) {
  if (g_tuning.split_rows_per_block > 0) return g_tuning.split_rows_per_block;
  const int64_t r = (rows + sm_count - 1) / sm_count;
  return static_cast<int32_t>(r < mla::kSplitAutoMaxRows ? r : mla::kSplitAutoMaxRows);
}

mla_status make_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* p) {
  const int64_t rows = T * (H + 1);
  const bool split = (flags & MLA_FLAG_FORCE_SPLIT)  ? true
                     : (flags & MLA_FLAG_FORCE_ROWS) ? false
                                                      : rows <= g_tuning.split_max_rows;
  p->sm_count = sm_count;
  if (split) {
    const int32_t rpb = split_rows(rows, sm_count);
    p->mode = MLA_MODE_SPLIT;
    p->rows_per_block = rpb;
    p->threads_per_block = mla::kSplitThreadsPerRow * rpb;
    p->blocks = (rows + rpb - 1) / rpb;
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
  if (t->split_rows_per_block > 0) {
    g_tuning.split_rows_per_block =
        t->split_rows_per_block < mla::kSplitMaxRowsPerBlock ? t->split_rows_per_block : mla::kSplitMaxRowsPerBlock;
  } else if (t->split_rows_per_block < 0) {
    g_tuning.split_rows_per_block = 0;  // back to the automatic choice
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
  a.pe_vec = aligned(q_pe, 4) && aligned(k_pe, 4) && (T == 1 || (q_pe_stride_t % 2 == 0 && k_pe_stride_t % 2 == 0)) &&
             (H == 1 || q_pe_stride_h % 2 == 0) && (!rope || aligned(cos_sin, 8));
  a.q_scale = q_scale;
  a.kv_scale = kv_scale;
  a.T = T;
  a.H = H;
  a.h_magic = H > 1 ? (UINT64_MAX / static_cast<uint64_t>(H)) + 1 : 0;
  {
    uint32_t sh = 0;  // ceil(log2 H)
    while ((INT64_C(1) << sh) < H) ++sh;
    a.h_magic32 = H > 1 ? static_cast<uint32_t>(((UINT64_C(1) << (31 + sh)) + static_cast<uint64_t>(H) - 1) /
                                                static_cast<uint64_t>(H))
                        : 0u;
    a.h_shift32 = H > 1 ? sh - 1 : 0u;
  }
  a.cache_rows = cache_rows;
  a.rows = T * (H + 1);
  a.q_out = static_cast<uint8_t*>(q_out);
  a.cache = static_cast<uint8_t*>(cache);
  a.status = status;

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
