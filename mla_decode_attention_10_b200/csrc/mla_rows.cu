// mla_rows.cu -- the large-batch (MLA_MODE_ROWS) kernel of the fused MLA
// decode epilogue: one warp per row, grid-stride over rows, each warp
// keeping its next rows in flight through a shared-memory ring.
//
// The rows of a call are the cache rows [0, T), then the query rows in q_out
// order (vLLM PR #54896 report, 实现拆解 items 1-3).  Warp w of the grid
// takes rows w, w + W, w + 2W, ... (W = all warps of the grid), so all warps
// walk one window of memory together.  Each warp owns kDepth row slots of
// 1152 bytes in shared memory.  While it converts row i, the 16-byte
// cp.async copies (the load/store unit's asynchronous path, L2 only) of rows
// i + 1 .. i + kDepth - 1 are in flight: the bytes in flight cost no
// registers, so every SM keeps over 100 KB of loads outstanding.  The
// token's position and slot are loaded two rows ahead and its cos/sin pair
// one row ahead, into registers.
//
// Converting row i: lane l takes nope chunks l and l + 32 (16 bytes each)
// and pe pair (l, l + 32) from its slot, rotates and encodes them, stores the
// nope chunks straight to global memory (16-byte bf16 or 8-byte e4m3 stores,
// 512 or 256 contiguous bytes per warp instruction), and writes its pe pair
// back into the slot, from which lanes 0..7 send the row's 64 or 128 pe
// bytes out as 8- or 16-byte stores.
//
// Query rows execute griddepcontrol.wait once, before the first copy of a
// query row is issued (the upstream kernel writes q_nope and q_pe); cache
// rows, slots, positions and table rows do not wait (实现拆解 item 2).  Every
// thread triggers its dependents after its last store (评论区精华: the early
// trigger was a race).

#include <cstdint>
#include <cuda_runtime.h>

#include "epilogue_device.cuh"
#include "mla_rows.h"
#include "mla_runtime.h"

namespace mla {
namespace rows {

constexpr int kDepth = 4;         // row slots per warp (kDepth - 1 rows ahead)
constexpr uint32_t kSlot = 1152;  // one row: 1024 nope bytes, then 128 pe bytes
// 5 blocks of 8 warps per SM: 40 warps, 184 KB of rings, 51 registers a thread
static_assert(kRowsMaxBlocksPerSm * kRowsMaxWarps * kDepth * kSlot <= 227 * 1024, "rings fit in shared memory");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// this thread's copies of all but its newest kDepth - 1 groups have landed
__device__ __forceinline__ void cp_async_wait_row() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kDepth - 1) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Where row g comes from and goes to.
struct RowRef {
  const uint16_t* nope;
  const uint16_t* pe;
  int64_t t;  // token
  int64_t q;  // query row (q_out row), or -1 for a cache row
  bool valid;
};

__device__ __forceinline__ RowRef row_ref(const Args& a, int64_t g) {
  RowRef r;
  r.valid = g < a.rows;
  r.nope = nullptr;
  r.pe = nullptr;
  r.t = 0;
  r.q = -1;
  if (!r.valid) return r;
  if (g < a.T) {
    r.t = g;
    r.nope = a.kv_c + g * a.kv_st;
    r.pe = a.k_pe + g * a.kp_st;
  } else {
    r.q = g - a.T;
    r.t = div_heads(a, r.q);
    const int64_t h = r.q - r.t * a.H;
    r.nope = a.q_nope + r.t * a.qn_st + h * a.qn_sh;
    r.pe = a.q_pe + r.t * a.qp_st + h * a.qp_sh;
  }
  return r;
}

// Issue the copies of row r into `slot` (one commit group per lane, empty for
// a row past the end): nope chunks lane and lane + 32 and, when the pe row is
// on the 16-byte grid, its 8 chunks by lanes 0..7.
__device__ __forceinline__ void issue_row(const Args& a, const RowRef& r, uint32_t slot, int lane) {
  if (r.valid) {
    cp_async16(slot + 16u * lane, r.nope + 8 * lane);
    cp_async16(slot + 512u + 16u * lane, r.nope + 256 + 8 * lane);
    const bool vec = (r.q < 0) ? a.kpe_vec != 0 : a.qpe_vec != 0;
    if (vec && lane < 8) cp_async16(slot + 1024u + 16u * lane, r.pe + 8 * lane);
  }
  cp_async_commit();
}

// A row's token position (with RoPE) and cache slot (cache rows), loaded two
// rows ahead of their use.
struct Ahead {
  int64_t slot;
  int32_t pos;
};

template <bool ROPE>
__device__ __forceinline__ Ahead ahead_of(const Args& a, int64_t g) {
  Ahead x{-1, -1};
  if (g < a.rows) {
    const int64_t t = g < a.T ? g : div_heads(a, g - a.T);
    if (g < a.T) x.slot = __ldg(a.slots + t);
    if constexpr (ROPE) x.pos = __ldg(a.positions + t);
  }
  return x;
}

// (cos, sin) of pair `lane` at position p, or `on` false when p is out of range.
struct Rot {
  float c, s;
  bool on;
};

template <bool ROPE>
__device__ __forceinline__ Rot rotation_of(const Args& a, int32_t p, int lane) {
  Rot r{1.0f, 0.0f, false};
  if constexpr (ROPE) {
    if (p >= 0 && p < a.rope_rows) {
      const float* row = a.cos_sin + static_cast<int64_t>(p) * kPe;
      r.c = __ldg(row + lane);
      r.s = __ldg(row + kHalfPe + lane);
      r.on = true;
    }
  }
  return r;
}

// Convert the staged row and store it to `dst`: nope by every lane, pe by
// lanes 0..7 through the slot's pe area.
template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void emit_row(uint8_t* slot, const RowRef& r, bool pe_vec, const Rot& rot, uint8_t* dst,
                                         int lane, const Divisor& d) {
  const uint4 n0 = *reinterpret_cast<const uint4*>(slot + 16 * lane);
  const uint4 n1 = *reinterpret_cast<const uint4*>(slot + 512 + 16 * lane);
  uint32_t pe;
  if (pe_vec) {
    pe = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(slot + 1024 + 2 * lane)) |
         (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(slot + 1088 + 2 * lane)) << 16);
  } else {
    pe = static_cast<uint32_t>(__ldcg(r.pe + lane)) | (static_cast<uint32_t>(__ldcg(r.pe + kHalfPe + lane)) << 16);
  }
  float ya = bf16_lo(pe), yb = bf16_hi(pe);
  if (ROPE && rot.on) rope_pair(bf16_lo(pe), bf16_hi(pe), rot.c, rot.s, ya, yb);
  __syncwarp();  // every lane has read its pe pair: the pe area becomes the output staging
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(dst + 8 * lane) = chunk_to_e4m3<FAST>(n0, d);
    *reinterpret_cast<uint2*>(dst + 256 + 8 * lane) = chunk_to_e4m3<FAST>(n1, d);
    const uint32_t p = e4m3x2_of_f32<FAST>(ya, yb, d);
    slot[1024 + lane] = static_cast<uint8_t>(p & 0xffu);
    slot[1024 + kHalfPe + lane] = static_cast<uint8_t>((p >> 8) & 0xffu);
    __syncwarp();
    if (lane < 8)
      *reinterpret_cast<uint2*>(dst + kNope + 8 * lane) = *reinterpret_cast<const uint2*>(slot + 1024 + 8 * lane);
  } else {
    *reinterpret_cast<uint4*>(dst + 16 * lane) = n0;
    *reinterpret_cast<uint4*>(dst + 512 + 16 * lane) = n1;
    const uint32_t p = (ROPE && rot.on) ? pack_bf16x2(ya, yb) : pe;  // unrotated values keep their bits
    *reinterpret_cast<uint16_t*>(slot + 1024 + 2 * lane) = static_cast<uint16_t>(p & 0xffffu);
    *reinterpret_cast<uint16_t*>(slot + 1088 + 2 * lane) = static_cast<uint16_t>(p >> 16);
    __syncwarp();
    if (lane < 8)
      *reinterpret_cast<uint4*>(dst + 2 * kNope + 16 * lane) = *reinterpret_cast<const uint4*>(slot + 1024 + 16 * lane);
  }
}

template <bool QF8, bool KVF8, bool ROPE, bool FAST>
__device__ __forceinline__ void run(const Args& a, uint8_t* ring, const Divisor& dq, const Divisor& dk) {
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int64_t W = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const uint32_t ring_s = smem_u32(ring);
  bool waited = false;

  // prologue: rows 0 .. kDepth - 2 of this warp in flight; slot and position
  // of rows 0 and 1; rotation of row 0
#pragma unroll
  for (int k = 0; k < kDepth - 1; ++k) {
    const RowRef r = row_ref(a, first + k * W);
    if (!waited && r.valid && r.q >= 0) {
      pdl_wait();  // the query inputs come from the upstream kernel
      waited = true;
    }
    issue_row(a, r, ring_s + k * kSlot, lane);
  }
  Ahead x0 = ahead_of<ROPE>(a, first);
  Ahead x1 = ahead_of<ROPE>(a, first + W);
  Rot rot0 = rotation_of<ROPE>(a, x0.pos, lane);

  for (int64_t i = 0;; ++i) {
    const int64_t g = first + i * W;
    if (g >= a.rows) break;
    // ahead: copies of row i + kDepth - 1, slot and position of row i + 2, rotation of row i + 1
    const RowRef nxt = row_ref(a, g + (kDepth - 1) * W);
    if (!waited && nxt.valid && nxt.q >= 0) {
      pdl_wait();
      waited = true;
    }
    issue_row(a, nxt, ring_s + static_cast<uint32_t>((i + kDepth - 1) % kDepth) * kSlot, lane);
    const Ahead x2 = ahead_of<ROPE>(a, g + 2 * W);
    const Rot rot1 = rotation_of<ROPE>(a, x1.pos, lane);

    // row i
    const RowRef cur = row_ref(a, g);
    uint8_t* slot = ring + static_cast<uint32_t>(i % kDepth) * kSlot;
    uint8_t* dst = nullptr;
    if (cur.q < 0) {
      if (x0.slot >= 0 && x0.slot < a.cache_rows) {
        dst = a.cache + x0.slot * (KVF8 ? kRow : 2 * kRow);
      } else if (x0.slot >= a.cache_rows && lane == 0) {
        report(a.status, MLA_STATUS_SLOT_RANGE);
      }
      if (ROPE && !rot0.on && lane == 0) report(a.status, MLA_STATUS_POS_RANGE);
    } else {
      dst = a.q_out + cur.q * (QF8 ? kRow : 2 * kRow);
    }
    cp_async_wait_row();
    __syncwarp();  // every lane's copies of row i are visible to the warp
    if (dst != nullptr) {
      if (cur.q < 0) {
        emit_row<KVF8, ROPE, FAST>(slot, cur, a.kpe_vec != 0, rot0, dst, lane, dk);
      } else {
        emit_row<QF8, ROPE, FAST>(slot, cur, a.qpe_vec != 0, rot0, dst, lane, dq);
      }
    }
    __syncwarp();  // the slot is free for the copies issued next iteration
    x0 = x1;
    x1 = x2;
    rot0 = rot1;
  }
  cp_async_wait_all();  // nothing may land in the ring after the block ends
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(32 * kRowsMaxWarps, kRowsMaxBlocksPerSm) mla_epilogue_rows_kernel(const Args a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* ring = smem + (threadIdx.x >> 5) * (kDepth * kSlot);
  // scales are read before any wait; every row takes the corrected-
  // reciprocal quotient unless a scale is outside [2^-64, 2^64]
  const Divisor dq = divisor_of<QF8>(a.q_scale);
  const Divisor dk = divisor_of<KVF8>(a.kv_scale);
  if (dq.fast && dk.fast) {
    run<QF8, KVF8, ROPE, true>(a, ring, dq, dk);
  } else {
    run<QF8, KVF8, ROPE, false>(a, ring, dq, dk);
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

void rows_plan(int64_t rows, bool, bool, int32_t sm_count, int32_t blocks_per_sm, int32_t warps_per_block,
               mla_plan* p) {
  const int32_t w = warps_per_block < kRowsMaxWarps ? warps_per_block : kRowsMaxWarps;
  const int64_t need = (rows + w - 1) / w;
  const int32_t per_sm = blocks_per_sm < kRowsMaxBlocksPerSm ? blocks_per_sm : kRowsMaxBlocksPerSm;
  const int64_t cap = static_cast<int64_t>(sm_count) * per_sm;
  p->mode = MLA_MODE_ROWS;
  p->rows_per_block = 1;
  p->threads_per_block = 32 * w;
  p->blocks = need < cap ? need : cap;
}

mla_status rows_kernel(int flag_bits, int warps, const void** fn, size_t* smem_bytes) {
  *fn = rows::kKernels[flag_bits & 7];
  *smem_bytes = static_cast<size_t>(warps) * rows::kDepth * rows::kSlot;
  return MLA_OK;
}

}  // namespace mla
