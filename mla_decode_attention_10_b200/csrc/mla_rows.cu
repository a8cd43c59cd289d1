// mla_rows.cu -- the large-batch (MLA_MODE_ROWS) kernel of the fused MLA
// decode epilogue: a persistent, warp-specialised stream through shared
// memory.
//
// The rows of a call (cache rows [0, T), then the query rows in q_out order;
// vLLM PR #54896 report, 实现拆解 items 1-3) are cut into tiles of 32 rows,
// and tile i goes to block i mod grid, so all blocks walk memory together.
// Each block (one per SM) has
//   * one producer warp: lane l owns row l of a tile.  It loads the row's
//     slot and position one tile ahead, then moves the row's 1024 nope bytes,
//     its 128 pe bytes and (once per token per tile) the token's 256-byte
//     cos/sin row into a four-stage shared-memory ring with bulk async copies
//     (cp.async.bulk) that complete on the stage's mbarrier, plus a small
//     per-row record (destination, position, table slot).  Query rows'
//     copies start only after griddepcontrol.wait (the upstream kernel writes
//     q_nope and q_pe); cache rows, slots, positions and table rows do not
//     wait (实现拆解 item 2);
//   * W consumer warps: warp w takes rows w, w + W, ... of a tile.  Lane l
//     reads nope chunks l and l + 32 and pe pair (l, l + 32) from shared
//     memory, rotates and encodes them, writes the finished row back in place
//     (e4m3 rows shrink to 576 bytes; bf16 nope values are already final) and
//     one lane sends the row to q_out or to its cache slot with one bulk store
//     (cp.async.bulk.global.shared), so global memory sees whole 576- or
//     1152-byte row writes and no per-element stores.
// A stage is handed back to the producer once the bulk stores that read it
// have finished reading (one tile later, so those waits overlap the next
// tile's work).  Every wait is bounded: on timeout the block sets
// MLA_STATUS_TIMEOUT, stops issuing, waits (bounded) for its copies in flight
// and returns.  Every thread triggers its dependents after its last store has
// completed (评论区精华: the early trigger was a race).

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "epilogue_device.cuh"
#include "mla_rows.h"
#include "mla_runtime.h"

namespace mla {
namespace rows {

constexpr int kTile = 32;                            // rows per tile (one producer lane each)
constexpr int kStages = 4;                           // shared-memory ring
constexpr uint32_t kRowBytes = 1152;                 // one staged row: 1024 nope bytes, then 128 pe bytes
constexpr uint32_t kTabBytes = 256;                  // one cos/sin row
constexpr uint32_t kMetaBytes = 32;                  // one row record
constexpr uint32_t kStageRows = kTile * kRowBytes;   // 36864
constexpr uint32_t kStageTab = kTile * kTabBytes;    // 8192
constexpr uint32_t kStageBytes = kStageRows + kStageTab + kTile * kMetaBytes;  // 46080
constexpr uint32_t kWaitSpins = 1u << 24;

// Per-row record written by the producer lane (generic stores, published by
// the stage's mbarrier arrive).
struct Meta {
  uint8_t* dst;        // output row, or null: nothing to write
  const uint16_t* pe;  // the row's pe source (read from global when not staged)
  int32_t pos;         // token position when the row is rotated, else -1
  int32_t tab;         // tile row whose table slot holds the token's cos/sin row
  int64_t pad;
};
static_assert(sizeof(Meta) == kMetaBytes, "row record size");

struct Bars {
  uint64_t full[kStages];
  uint64_t empty[kStages];
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0u;
}

// Bounded wait for the phase of `parity`; false on timeout or when another
// role has set the block's abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag) {
  for (uint32_t i = 0; i < kWaitSpins; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag != 0u) return false;
  }
  return false;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void bulk_store(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all_but_one() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void abort_block(volatile uint32_t* abort_flag, int32_t* status) {
  *abort_flag = 1u;
  report(status, MLA_STATUS_TIMEOUT);
}

// Slot (cache rows) and position of the token of global row g, loaded one
// tile ahead of their use.
struct Ahead {
  int64_t slot;
  int32_t pos;
};

template <bool ROPE>
__device__ __forceinline__ Ahead load_ahead(const Args& a, int64_t g) {
  Ahead r{-1, 0};
  if (g < a.rows) {
    const int64_t t = g < a.T ? g : div_heads(a, g - a.T);
    if (g < a.T) r.slot = __ldg(a.slots + t);
    if constexpr (ROPE) r.pos = __ldg(a.positions + t);
  }
  return r;
}

// ------------------------------------------------------------------------------------
// producer warp
// ------------------------------------------------------------------------------------

template <bool QF8, bool KVF8, bool ROPE>
__device__ __forceinline__ void produce(const Args& a, uint8_t* smem, const Bars& bars, int64_t tiles,
                                        volatile uint32_t* abort_flag) {
  const int lane = static_cast<int>(threadIdx.x) & 31;
  const int64_t step = gridDim.x;
  bool waited = false;
  int64_t k = 0;
  Ahead cur = load_ahead<ROPE>(a, static_cast<int64_t>(blockIdx.x) * kTile + lane);
  for (int64_t tile = blockIdx.x; tile < tiles; tile += step, ++k) {
    const Ahead nxt = load_ahead<ROPE>(a, (tile + step) * kTile + lane);
    const int st = static_cast<int>(k % kStages);
    uint8_t* stage = smem + st * kStageBytes;
    const uint32_t full = smem_u32(&bars.full[st]);
    const bool ready =
        k < kStages || mbar_wait(smem_u32(&bars.empty[st]), static_cast<uint32_t>((k / kStages - 1) & 1), abort_flag);
    if (!__all_sync(0xffffffffu, ready)) {  // the warp decides together
      if (lane == 0) abort_block(abort_flag, a.status);
      break;
    }

    // the row of this lane
    const int64_t g = tile * kTile + lane;
    const bool valid = g < a.rows;
    const bool is_cache = g < a.T;
    int64_t t = 0, q = 0;
    const uint16_t* nope = nullptr;
    const uint16_t* pe = nullptr;
    uint8_t* dst = nullptr;
    bool pe_staged = false;
    int32_t tab = lane;
    if (valid) {
      if (is_cache) {
        t = g;
        nope = a.kv_c + t * a.kv_st;
        pe = a.k_pe + t * a.kp_st;
        pe_staged = a.kpe_vec != 0;
        if (cur.slot >= 0 && cur.slot < a.cache_rows) {
          dst = a.cache + cur.slot * (KVF8 ? kRow : 2 * kRow);
        } else if (cur.slot >= a.cache_rows) {
          report(a.status, MLA_STATUS_SLOT_RANGE);
        }
      } else {
        q = g - a.T;
        t = div_heads(a, q);
        const int64_t h = q - t * a.H;
        nope = a.q_nope + t * a.qn_st + h * a.qn_sh;
        pe = a.q_pe + t * a.qp_st + h * a.qp_sh;
        pe_staged = a.qpe_vec != 0;
        dst = a.q_out + q * (QF8 ? kRow : 2 * kRow);
        tab = h < lane ? lane - static_cast<int32_t>(h) : 0;  // first row of this token in the tile
      }
    }
    bool rot = false;
    if constexpr (ROPE) {
      rot = valid && cur.pos >= 0 && cur.pos < a.rope_rows;
      if (valid && is_cache && !rot) report(a.status, MLA_STATUS_POS_RANGE);
    }
    const bool copy_tab = rot && a.tab_vec && tab == lane;
    const uint32_t bytes = (valid ? 1024u : 0u) + (valid && pe_staged ? 128u : 0u) + (copy_tab ? kTabBytes : 0u);
    const uint32_t total = __reduce_add_sync(0xffffffffu, bytes);

    // query rows read what the upstream kernel writes: wait for it once
    if (!waited && (tile * kTile + kTile - 1) >= a.T) {
      pdl_wait();
      waited = true;
    }
    if (lane == 0) mbar_expect_tx(full, total);
    Meta m;
    m.dst = dst;
    m.pe = pe;
    m.pos = rot ? cur.pos : -1;
    m.tab = tab;
    m.pad = 0;
    reinterpret_cast<Meta*>(stage + kStageRows + kStageTab)[lane] = m;
    __syncwarp();
    if (valid) {
      const uint32_t row = smem_u32(stage + lane * kRowBytes);
      bulk_load(row, nope, 1024u, full);
      if (pe_staged) bulk_load(row + 1024u, pe, 128u, full);
    }
    if (copy_tab) bulk_load(smem_u32(stage + kStageRows + lane * kTabBytes), a.cos_sin + cur.pos * kPe, kTabBytes, full);
    __syncwarp();
    if (lane == 0) mbar_arrive(full);
    cur = nxt;
  }

  // every copy issued must land before the block may end: wait (bounded) for
  // the last kStages tiles' stages
  const int64_t issued = k;
  for (int64_t j = issued > kStages ? issued - kStages : 0; j < issued; ++j) {
    const uint32_t full = smem_u32(&bars.full[j % kStages]);
    for (uint32_t i = 0; i < kWaitSpins && !mbar_try_wait(full, static_cast<uint32_t>((j / kStages) & 1)); ++i) {
    }
  }
}

// ------------------------------------------------------------------------------------
// consumer warps
// ------------------------------------------------------------------------------------

// One staged row: rotate and encode it, write the output over the row in
// shared memory (e4m3: 576 bytes from the start; bf16: only the pe part
// changes) and send it to `m.dst` with one bulk store issued by lane 0.
// Lane l handles nope chunks l and l + 32 and pe pair (l, l + 32).
template <bool FP8, bool ROPE, bool FAST>
__device__ __forceinline__ void convert_row(uint8_t* row, const uint8_t* tab, const Meta& m, bool pe_staged,
                                            bool tab_staged, const Args& a, int lane, const Divisor& d) {
  // 1. every input of the lane into registers
  uint4 n0 = make_uint4(0, 0, 0, 0), n1 = n0;
  if constexpr (FP8) {
    n0 = *reinterpret_cast<const uint4*>(row + 16 * lane);
    n1 = *reinterpret_cast<const uint4*>(row + 512 + 16 * lane);
  }
  uint32_t pe;
  if (pe_staged) {
    pe = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(row + 1024 + 2 * lane)) |
         (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(row + 1088 + 2 * lane)) << 16);
  } else {
    pe = static_cast<uint32_t>(__ldcg(m.pe + lane)) | (static_cast<uint32_t>(__ldcg(m.pe + kHalfPe + lane)) << 16);
  }
  bool on = false;
  float c = 1.0f, s = 0.0f;
  if constexpr (ROPE) {
    if (m.pos >= 0) {
      on = true;
      if (tab_staged) {
        c = reinterpret_cast<const float*>(tab)[lane];
        s = reinterpret_cast<const float*>(tab)[kHalfPe + lane];
      } else {
        const float* tr = a.cos_sin + static_cast<int64_t>(m.pos) * kPe;
        c = __ldg(tr + lane);
        s = __ldg(tr + kHalfPe + lane);
      }
    }
  }
  // 2. the pe pair
  float ya = bf16_lo(pe), yb = bf16_hi(pe);
  if (ROPE && on) rope_pair(bf16_lo(pe), bf16_hi(pe), c, s, ya, yb);
  __syncwarp();  // every lane has read the row before any output overwrites it
  // 3. the output row over the staged row
  if constexpr (FP8) {
    *reinterpret_cast<uint2*>(row + 8 * lane) = chunk_to_e4m3<FAST>(n0, d);
    *reinterpret_cast<uint2*>(row + 256 + 8 * lane) = chunk_to_e4m3<FAST>(n1, d);
    const uint32_t p = e4m3x2_of_f32<FAST>(ya, yb, d);
    row[kNope + lane] = static_cast<uint8_t>(p & 0xffu);
    row[kNope + kHalfPe + lane] = static_cast<uint8_t>((p >> 8) & 0xffu);
  } else if ((ROPE && on) || !pe_staged) {
    const uint32_t p = (ROPE && on) ? pack_bf16x2(ya, yb) : pe;  // unrotated values keep their bits
    *reinterpret_cast<uint16_t*>(row + 1024 + 2 * lane) = static_cast<uint16_t>(p & 0xffffu);
    *reinterpret_cast<uint16_t*>(row + 1088 + 2 * lane) = static_cast<uint16_t>(p >> 16);
  }
  fence_proxy_async();  // this lane's shared-memory writes are visible to the bulk copy
  __syncwarp();
  if (lane == 0) bulk_store(m.dst, smem_u32(row), FP8 ? static_cast<uint32_t>(kRow) : 2u * kRow);
}

template <bool QF8, bool KVF8, bool ROPE, bool FAST>
__device__ __forceinline__ void consume(const Args& a, uint8_t* smem, const Bars& bars, int64_t tiles, int warps,
                                        int w, volatile uint32_t* abort_flag, const Divisor& dq, const Divisor& dk) {
  const int lane = static_cast<int>(threadIdx.x) & 31;
  // query pe rows off the 16-byte grid are read here, from global memory:
  // they come from the upstream kernel, so wait for it first
  if (!a.qpe_vec) pdl_wait();
  int64_t k = 0;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++k) {
    const int st = static_cast<int>(k % kStages);
    uint8_t* stage = smem + st * kStageBytes;
    const bool ready = mbar_wait(smem_u32(&bars.full[st]), static_cast<uint32_t>((k / kStages) & 1), abort_flag);
    if (!__all_sync(0xffffffffu, ready)) {  // the warp decides together
      if (lane == 0) abort_block(abort_flag, a.status);
      break;
    }
    const Meta* meta = reinterpret_cast<const Meta*>(stage + kStageRows + kStageTab);
    for (int r = w; r < kTile; r += warps) {
      const Meta m = meta[r];
      if (m.dst == nullptr) continue;
      uint8_t* row = stage + r * kRowBytes;
      const uint8_t* tab = stage + kStageRows + m.tab * kTabBytes;
      if (tile * kTile + r < a.T) {
        convert_row<KVF8, ROPE, FAST>(row, tab, m, a.kpe_vec != 0, a.tab_vec != 0, a, lane, dk);
      } else {
        convert_row<QF8, ROPE, FAST>(row, tab, m, a.qpe_vec != 0, a.tab_vec != 0, a, lane, dq);
      }
    }
    if (lane == 0) {
      bulk_commit();
      // the previous tile's stores have read their rows: hand its stage back
      if (k > 0) {
        bulk_wait_read_all_but_one();
        mbar_arrive(smem_u32(&bars.empty[(k - 1) % kStages]));
      }
    }
    __syncwarp();
  }
  if (lane == 0) bulk_wait_all();  // every store of this warp has completed
}

template <bool QF8, bool KVF8, bool ROPE>
__global__ void __launch_bounds__(32 * (1 + kRowsMaxConsumerWarps), 1) mla_epilogue_rows_kernel(const Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t abort_flag;
  const int warp = static_cast<int>(threadIdx.x) >> 5;
  const int warps = static_cast<int>(blockDim.x >> 5) - 1;  // consumer warps
  const int64_t tiles = (a.rows + kTile - 1) / kTile;
  if (threadIdx.x == 0) {
    abort_flag = 0u;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&bars.full[s]), 1);
      mbar_init(smem_u32(&bars.empty[s]), static_cast<uint32_t>(warps));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {
    produce<QF8, KVF8, ROPE>(a, smem, bars, tiles, &abort_flag);
  } else {
    // scales are read before any wait; every row takes the corrected-
    // reciprocal quotient unless a scale is outside [2^-64, 2^64]
    const Divisor dq = divisor_of<QF8>(a.q_scale);
    const Divisor dk = divisor_of<KVF8>(a.kv_scale);
    if (dq.fast && dk.fast) {
      consume<QF8, KVF8, ROPE, true>(a, smem, bars, tiles, warps, warp - 1, &abort_flag, dq, dk);
    } else {
      consume<QF8, KVF8, ROPE, false>(a, smem, bars, tiles, warps, warp - 1, &abort_flag, dq, dk);
    }
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

// whether kernel k has its shared-memory opt-in on device `dev`
std::atomic<bool> g_smem_ready[kMaxDevices][8];

}  // namespace rows

void rows_plan(int64_t rows, bool, bool, int32_t sm_count, int32_t blocks_per_sm, int32_t warps_per_block,
               mla_plan* p) {
  const int64_t tiles = (rows + rows::kTile - 1) / rows::kTile;
  const int64_t cap = static_cast<int64_t>(sm_count) * (blocks_per_sm < kRowsMaxBlocksPerSm ? blocks_per_sm
                                                                                            : kRowsMaxBlocksPerSm);
  p->mode = MLA_MODE_ROWS;
  p->rows_per_block = rows::kTile;
  p->threads_per_block = 32 * (1 + warps_per_block);
  p->blocks = tiles < cap ? tiles : cap;
}

mla_status rows_kernel(int flag_bits, int dev, const void** fn, size_t* smem_bytes) {
  const int k = flag_bits & 7;
  *fn = rows::kKernels[k];
  *smem_bytes = rows::kStages * rows::kStageBytes;
  if (!rows::g_smem_ready[dev][k].load(std::memory_order_acquire)) {
    // idempotent: two threads racing here both set the same attribute
    const cudaError_t e =
        cudaFuncSetAttribute(*fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(*smem_bytes));
    if (e != cudaSuccess) return cuda_failure(e);
    rows::g_smem_ready[dev][k].store(true, std::memory_order_release);
  }
  return MLA_OK;
}

}  // namespace mla
