// mla_rows.cu -- the large-batch (MLA_MODE_ROWS) kernel of the fused MLA
// decode epilogue: a fixed group of lanes per row, grid-stride over rows, the
// grid sized to the resident blocks on every SM.
//
// The rows of a call are the cache rows [0, T), then the query rows in q_out
// order (vLLM PR #54896 report, 实现拆解 items 1-3).  A warp converts 32 / L
// adjacent rows per trip (L lanes each) and then moves on by the number of
// warps in the grid, so all warps walk one window of memory together.  Lane l
// of a row moves nope chunks l + k L (16 bytes each) and rotates the pe pairs
// (i, i + 32) for i = l + k L, or, with L = 16 and the pe rows and the table
// aligned, for i = 2l and 2l + 1 (vector loads and stores; the launcher sets
// pe_vec).  With an e4m3 output L = 16: the kernel is
// bound by instruction issue (measured on B200), and two rows per warp trip
// halve the per-row instructions (addresses, slot, position, table row,
// checks) while the e4m3 arithmetic stays spread over all 32 lanes.  bf16
// outputs, bound by memory, keep L = 32 (one row per warp).
//
// Query rows execute griddepcontrol.wait once, before their first read of
// q_nope / q_pe (the upstream kernel writes them); cache rows, slots,
// positions and table rows do not wait (实现拆解 item 2).  Every thread
// triggers its dependents after its last store (评论区精华: the early trigger
// was a race).

#include <climits>
#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>

#include "epilogue_device.cuh"
#include "mla_rows.h"
#include "mla_runtime.h"

namespace mla {
namespace rows {

// Lanes per row and resident 256-thread blocks per SM the kernel is compiled
// for.  e4m3 outputs: 16 lanes per row at 4 blocks (64 registers; measured on
// B200 at T=8192, H=16: 40.1 us against 42.5 for one warp per row at 6
// blocks and 41.0 at 5).  bf16 outputs: one warp per row at 5 blocks (44
// registers; 49.9 us at T=1024, H=128 against 53.4 for 16 lanes per row).
__host__ __device__ constexpr int rows_lanes_per_row(bool qf8, bool kvf8) { return (qf8 || kvf8) ? 16 : 32; }
constexpr int rows_blocks_per_sm(bool qf8, bool kvf8) { return (qf8 || kvf8) ? 4 : 5; }
static_assert(rows_blocks_per_sm(true, true) <= kRowsMaxBlocksPerSm, "tuning limit covers the resident count");

// q / H for the row loop.  64-bit rows: one multiply-high by ceil(2^64 / H)
// (div_heads).  32-bit rows (every call: T * (H + 1) < 2^31): with
// 2^(s-1) < H <= 2^s and M = ceil(2^(31+s) / H) < 2^32 (h_magic32, set by
// the host), floor(q M / 2^(31+s)) = floor(q / H) for 0 <= q < 2^31
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994): one 32-bit multiply-high and a shift.
__device__ __forceinline__ uint32_t div_h(const Args& a, uint32_t q) {
  return a.h_magic32 == 0u ? q : __umulhi(q, a.h_magic32) >> a.h_shift32;
}
__device__ __forceinline__ int64_t div_h(const Args& a, int64_t q) { return div_heads(a, q); }

// Idx: the integer type of the row loop.  e4m3 outputs use 32 bits, unsigned
// so that the trip counter times rows per trip cannot wrap (rows < 2^31):
// the e4m3 kernel is bound by instruction issue, and 32-bit indexing saves a
// tenth of its instructions (measured on B200: 47.2 -> 44.2 us at T=8192,
// H=16); bf16 outputs, bound by memory, keep 64 bits (2% faster there).
// VEC (16 lanes per row, pe rows and table aligned): lane l takes the RoPE
// pairs 2l and 2l + 1 with one 4-byte load per pe half, one 8-byte load each
// of cos and sin, and one 2- or 4-byte store per pe half (store_pe2);
// otherwise lane l takes pairs l + k L, one 2-byte load and one store each.
template <int L, bool VEC, typename Idx, bool QF8, bool KVF8, bool ROPE, bool FAST>
__device__ __forceinline__ void rows_body(const Args& a, const Divisor& dq, const Divisor& dk) {
  static_assert(!VEC || L == 16, "two pairs per lane cover a row at 16 lanes");
  constexpr int kRowsPerTrip = 32 / L, kChunks = 64 / L, kPairs = 32 / L;
  const int ll = threadIdx.x & (L - 1);
  const Idx sub = static_cast<Idx>((threadIdx.x & 31) / L);
  const Idx H = static_cast<Idx>(a.H);
  const Idx T = static_cast<Idx>(a.T);
  const Idx rows = static_cast<Idx>(a.rows);
  const int32_t rope_rows = a.rope_rows < INT32_MAX ? static_cast<int32_t>(a.rope_rows) : INT32_MAX;
  const Idx warps = static_cast<Idx>(gridDim.x) * static_cast<Idx>(blockDim.x >> 5);
  const Idx wid = static_cast<Idx>(blockIdx.x) * static_cast<Idx>(blockDim.x >> 5) + static_cast<Idx>(threadIdx.x >> 5);
  bool waited = false;

  for (Idx trip = wid; trip * kRowsPerTrip < rows; trip += warps) {
    const Idx g = trip * kRowsPerTrip + sub;
    if (g >= rows) continue;
    // 1. addresses, slot and rotation: nothing here depends on the upstream kernel
    const bool is_cache = g < T;
    Idx t;
    const uint16_t* nope;
    const uint16_t* pe;
    uint8_t* dst = nullptr;
    if (is_cache) {
      t = g;
      nope = a.kv_c + static_cast<int64_t>(t) * a.kv_st;
      pe = a.k_pe + static_cast<int64_t>(t) * a.kp_st;
      const int64_t slot = __ldg(a.slots + t);
      if (slot >= 0 && slot < a.cache_rows) {
        dst = a.cache + slot * (KVF8 ? kRow : 2 * kRow);
      } else if (slot >= a.cache_rows && ll == 0) {
        report(a.status, MLA_STATUS_SLOT_RANGE);
      }
    } else {
      const Idx q = g - T;
      t = div_h(a, q);
      const Idx h = q - t * H;
      nope = a.q_nope + static_cast<int64_t>(t) * a.qn_st + static_cast<int64_t>(h) * a.qn_sh;
      pe = a.q_pe + static_cast<int64_t>(t) * a.qp_st + static_cast<int64_t>(h) * a.qp_sh;
      dst = a.q_out + static_cast<int64_t>(q) * (QF8 ? kRow : 2 * kRow);
    }
    Rot rot[kPairs];
#pragma unroll
    for (int k = 0; k < kPairs; ++k) rot[k] = Rot{1.0f, 0.0f, false};
    if constexpr (ROPE) {
      const int32_t pos = __ldg(a.positions + t);
      if (pos >= 0 && pos < rope_rows) {
        const float* row = a.cos_sin + static_cast<int64_t>(pos) * kPe;
        if constexpr (VEC) {
          const float2 c = __ldg(reinterpret_cast<const float2*>(row) + ll);
          const float2 sn = __ldg(reinterpret_cast<const float2*>(row + kHalfPe) + ll);
          rot[0] = Rot{c.x, sn.x, true};
          rot[1] = Rot{c.y, sn.y, true};
        } else {
#pragma unroll
          for (int k = 0; k < kPairs; ++k) {
            rot[k].c = __ldg(row + ll + k * L);
            rot[k].s = __ldg(row + kHalfPe + ll + k * L);
            rot[k].on = true;
          }
        }
      }
      if (is_cache && ll == 0 && !rot[0].on) report(a.status, MLA_STATUS_POS_RANGE);
    }

    // 2. query rows read what the upstream kernel wrote: wait for it once
    if (!is_cache && !waited) {
      pdl_wait();
      waited = true;
    }

    // 3. the row's loads, then 4. convert and store
    uint4 n[kChunks];
    uint32_t p[kPairs];  // VEC: p[0] = pe[2l], pe[2l+1]; p[1] = pe[2l+32], pe[2l+33]
#pragma unroll
    for (int k = 0; k < kChunks; ++k) n[k] = ld_chunk(nope, ll + k * L);
    if constexpr (VEC) {
      p[0] = __ldcg(reinterpret_cast<const uint32_t*>(pe) + ll);
      p[1] = __ldcg(reinterpret_cast<const uint32_t*>(pe + kHalfPe) + ll);
    } else {
#pragma unroll
      for (int k = 0; k < kPairs; ++k) p[k] = ld_pair(pe, ll + k * L);
    }
    if (dst == nullptr) continue;
    if (is_cache) {
#pragma unroll
      for (int k = 0; k < kChunks; ++k) store_nope<KVF8, FAST>(dst, ll + k * L, n[k], dk);
      if constexpr (VEC) {
        store_pe2<KVF8, ROPE, FAST>(dst, 2 * ll, p[0], p[1], rot[0], rot[1], dk);
      } else {
#pragma unroll
        for (int k = 0; k < kPairs; ++k) store_pe<KVF8, ROPE, FAST>(dst, ll + k * L, p[k], rot[k], dk);
      }
    } else {
#pragma unroll
      for (int k = 0; k < kChunks; ++k) store_nope<QF8, FAST>(dst, ll + k * L, n[k], dq);
      if constexpr (VEC) {
        store_pe2<QF8, ROPE, FAST>(dst, 2 * ll, p[0], p[1], rot[0], rot[1], dq);
      } else {
#pragma unroll
        for (int k = 0; k < kPairs; ++k) store_pe<QF8, ROPE, FAST>(dst, ll + k * L, p[k], rot[k], dq);
      }
    }
  }
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(32 * kRowsMaxWarps, rows_blocks_per_sm(QF8, KVF8)) mla_epilogue_rows_kernel(const Args a) {
  // scales are read before any wait; the whole body takes the corrected-
  // reciprocal quotient unless a scale is outside [2^-64, 2^64]
  Divisor dq{}, dk{};
  dq.fast = dk.fast = true;
  if constexpr (QF8) dq = make_divisor(__ldg(a.q_scale));
  if constexpr (KVF8) dk = make_divisor(__ldg(a.kv_scale));
  using Idx = std::conditional_t<QF8 || KVF8, uint32_t, int64_t>;
  constexpr int L = rows_lanes_per_row(QF8, KVF8);
  constexpr bool kCanVec = L == 16;
  if (dq.fast && dk.fast) {
    if (kCanVec && a.pe_vec) {
      rows_body<L, kCanVec, Idx, QF8, KVF8, ROPE, true>(a, dq, dk);
    } else {
      rows_body<L, false, Idx, QF8, KVF8, ROPE, true>(a, dq, dk);
    }
  } else {
    rows_body<L, false, Idx, QF8, KVF8, ROPE, false>(a, dq, dk);
  }
  pdl_trigger();
}

template <int F>
const void* kernel_for() {
  return reinterpret_cast<const void*>(
      &mla_epilogue_rows_kernel<(F & MLA_FLAG_Q_FP8) != 0, (F & MLA_FLAG_KV_FP8) != 0, (F & MLA_FLAG_ROPE) != 0>);
}

const void* const kKernels[8] = {kernel_for<0>(), kernel_for<1>(), kernel_for<2>(), kernel_for<3>(),
                                 kernel_for<4>(), kernel_for<5>(), kernel_for<6>(), kernel_for<7>()};

}  // namespace rows

void rows_plan(int64_t rows, bool qf8, bool kvf8, int32_t sm_count, int32_t blocks_per_sm, int32_t warps_per_block,
               mla_plan* p) {
  const int32_t w = warps_per_block < kRowsMaxWarps ? warps_per_block : kRowsMaxWarps;
  const int64_t per_block = static_cast<int64_t>(w) * (32 / rows::rows_lanes_per_row(qf8, kvf8));
  const int64_t need = (rows + per_block - 1) / per_block;
  const int32_t resident = rows::rows_blocks_per_sm(qf8, kvf8);
  const int32_t per_sm = blocks_per_sm < resident ? blocks_per_sm : resident;
  const int64_t cap = static_cast<int64_t>(sm_count) * per_sm;
  p->mode = MLA_MODE_ROWS;
  p->rows_per_block = 32 / rows::rows_lanes_per_row(qf8, kvf8);
  p->threads_per_block = 32 * w;
  p->blocks = need < cap ? need : cap;
}

mla_status rows_kernel(int flag_bits, int, const void** fn, size_t* smem_bytes) {
  *fn = rows::kKernels[flag_bits & 7];
  *smem_bytes = 0;
  return MLA_OK;
}

}  // namespace mla
