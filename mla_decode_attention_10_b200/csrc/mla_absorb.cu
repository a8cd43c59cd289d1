// mla_absorb.cu -- latent query rows straight from the absorption product, on
// the tcgen05 tensor cores (contract in mla_absorb.h).
//
// A persistent kernel, one CTA per SM, over 128-token x 256-column tiles.
// When the 2H (head, column half) pairs fit the grid, each pair gets
// grid / 2H CTAs that take every (grid / 2H)-th token tile of it, and the
// grid % 2H remaining CTAs share out the last token tiles of every pair: a
// CTA loads its weights once, and the running CTAs read all heads of the
// same token tiles together, which keeps DRAM pages open (measured on B200
// at T=8192, H=16, e4m3: 36.6 -> 34.9 us).  Otherwise each CTA takes a
// contiguous run of tiles in (head, column half, token tile) order.  Its
// warps have roles:
//   * warp 0 (TMA): per tile, the A tile (q_nope_c: 128 tokens x 128) into a
//     two-stage ring and, when the (head, column half) changes, the B tile
//     (w_uk: 256 latent rows x 128), both with the 128-byte swizzle; the
//     weights before waiting for the upstream grid, the queries after;
//   * warp 1 (MMA): allocates 512 TMEM columns and per tile issues eight
//     M=128, N=256, K=16 tcgen05.mma (bf16 in, fp32 accumulate) into one of
//     two 256-column accumulators, committing to the A stage's "empty" and
//     the accumulator's "full" barrier;
//   * warps 2..9 (epilogue): the warp of TMEM lane quarter w mod 4 and column
//     half (w - 2) / 4 reads its 32 tokens x 128 columns with tcgen05.ld,
//     encodes them (bf16, or e4m3 of x / scale) into a staging tile with the
//     128-byte swizzle, frees the accumulator, and one thread per half sends
//     each 128-byte column slab out with one bulk tensor store, so HBM sees
//     whole-line writes.  An e4m3 tile (32 KB) uses half of the 64 KB staging
//     area, alternating halves from tile to tile, so a tile waits only for
//     the stores of two tiles back;
//   * warps 10..15 (rotary): the 64 pe values of every head of the CTA's
//     share of the tokens, two threads per (token, head), every load issued
//     before any is used; consecutive threads take consecutive heads of one
//     token, so a token's table row is read once per warp and its q_pe rows
//     as one contiguous run.  Six rotary warps fill the 64 K registers at
//     128 a thread (measured on B200 at T=8192, H=16, e4m3: 41.2 -> 36.7 us
//     with the staging halves; either change alone gains at most 2%).
// The loads of tile i+1, its MMAs and the epilogue of tile i overlap.  Every
// wait is bounded: on timeout the kernel sets a status bit, every role stops,
// the copies in flight are waited for (bounded), TMEM is freed and the kernel
// returns.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <climits>
#include <cstdint>

#include "latent_math.cuh"
#include "mla_absorb.h"
#include "mla_runtime.h"

namespace mla {
namespace absorb {

constexpr int kM = 128;          // tokens per tile (UMMA M)
constexpr int kN = 256;          // latent columns per tile (UMMA N)
constexpr int kK = 128;          // contraction (nope head dim before absorption)
constexpr int kNope = 512;
constexpr int kPe = 64;
constexpr int kHalfPe = 32;
constexpr int kRow = 576;
constexpr int kTmaWarp = 0, kMmaWarp = 1, kEpiWarp0 = 2, kEpiWarps = 8, kPeWarp0 = 10, kPeWarps = 6;
constexpr int kThreads = 32 * (kPeWarp0 + kPeWarps);  // 512: the register file at 128 a thread
constexpr int kStages = 2;                            // A ring
constexpr uint32_t kSlabA = kM * 64 * 2;     // one 64-wide column slab of A: 16 KB
constexpr uint32_t kSlabB = kN * 64 * 2;     // one 64-wide column slab of B: 32 KB
constexpr uint32_t kSlabC = kM * 128;        // one 128-byte column slab of the output tile: 16 KB
constexpr uint32_t kABytes = 2 * kSlabA;                 // 32 KB
constexpr uint32_t kBBytes = 2 * kSlabB;                 // 64 KB
constexpr uint32_t kCBytes = 4 * kSlabC;                 // output staging, 64 KB
constexpr uint32_t kSmemBytes = kBBytes + kStages * kABytes + kCBytes + 1024;
constexpr uint32_t kTmemCols = 512;  // two 256-column accumulators
constexpr uint32_t kWaitSpins = 1u << 24;

struct Params {
  const uint16_t* q_pe;
  int64_t qp_st, qp_sh;
  const int32_t* positions;
  const float* cos_sin;
  int64_t rope_rows;
  const float* q_scale;
  int32_t T, H;
  uint8_t* q_out;
  int32_t* status;
  int32_t pe_vec;   // q_pe rows may be read as 16-byte vectors
  int32_t tab_vec;  // cos_sin rows may be read as 16-byte vectors
  int32_t strided;    // 2H <= grid: the per-(head, half) assignment above, else contiguous runs
  int32_t per_combo;  // main CTAs per (head, half): CTA c < per_combo * 2H takes pair c mod 2H
  int32_t tail;       // last token tiles of every pair, shared out to the CTAs past the main ones
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void report(int32_t* status, int32_t bit) {
  if (status != nullptr) atomicOr(status, bit);
}

__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitSpins; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored as 128-byte
// swizzled rows (8-row groups 1024 bytes apart): start address, leading byte
// offset 16 (unused for this layout), stride byte offset 1024, descriptor
// version 1, layout "128-byte swizzle" (2).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr) {
  return static_cast<uint64_t>((addr >> 4) & 0x3fffu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kN >> 3) << 17) | ((kM >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(kInstrDesc), "r"(accumulate)
      : "memory");
}

// tcgen05.ld of 32 columns of this warp's 32 TMEM lanes, then its wait; the
// wait names the loaded registers, so no use of them can be scheduled
// before it
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]), "+r"(v[6]), "+r"(v[7]),
                 "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]), "+r"(v[12]), "+r"(v[13]), "+r"(v[14]),
                 "+r"(v[15]), "+r"(v[16]), "+r"(v[17]), "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]),
                 "+r"(v[22]), "+r"(v[23]), "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]),
                 "+r"(v[29]), "+r"(v[30]), "+r"(v[31])
               :
               : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 32 accumulator values (columns col..col+31 of tile row r), encoded, into
// the output staging tile: 128-byte column slabs of 128 rows each
// (kSlabCols columns), with the 128-byte swizzle the bulk tensor store
// expects (16-byte piece j of row r at position j ^ (r mod 8)).  Eight
// consecutive rows thus cover all 32 banks for one piece index.
template <bool QF8, bool FAST>
__device__ __forceinline__ void stage_chunk(uint32_t sC, int r, int col, const uint32_t (&v)[32], const Divisor& d) {
  constexpr int kSlabCols = QF8 ? 128 : 64;
  const uint32_t rowbase = sC + static_cast<uint32_t>(col / kSlabCols) * kSlabC + static_cast<uint32_t>(r) * 128u;
  const uint32_t j0 = static_cast<uint32_t>((col % kSlabCols) * (QF8 ? 1 : 2) / 16);
  const uint32_t sw = static_cast<uint32_t>(r & 7);
  if constexpr (QF8) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = e4m3x2_of_f32<FAST>(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), d);
      const uint32_t hi = e4m3x2_of_f32<FAST>(__uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]), d);
      w[i] = lo | (hi << 16);
    }
#pragma unroll
    for (int q = 0; q < 2; ++q)
      st_shared_v4(rowbase + (((j0 + q) ^ sw) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
#pragma unroll
    for (int q = 0; q < 4; ++q)
      st_shared_v4(rowbase + (((j0 + q) ^ sw) << 4), w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// The 64 rotary values of one (token, head) row, half of them: token
// m0 + 64 nt + tid / 2, rotation pairs (i, i+32) for i in 16 (tid & 1) ..
// 16 (tid & 1) + 15.  The thread issues all of its loads (its q_pe values and
// its cos and sin entries, as 16-byte vectors when the host found them
// aligned) before it uses any: about two memory round trips (position, then
// table).
template <bool QF8, bool ROPE, bool FAST>
__device__ __forceinline__ void pe_part(const Params& p, int m0, int nt, int h, int tid, const Divisor& d) {
  const int t = m0 + 64 * nt + (tid >> 1);
  if (t >= p.T) return;
  const int i0 = (tid & 1) * 16;  // first rotation pair of this thread
  const uint16_t* pe = p.q_pe + static_cast<int64_t>(t) * p.qp_st + static_cast<int64_t>(h) * p.qp_sh;
  int32_t pos = 0;
  if constexpr (ROPE) pos = __ldg(p.positions + t);
  uint32_t ra[8], rb[8];  // bf16 pairs: first-half values a_i and second-half values b_i = pe[i + 32]
  if (p.pe_vec) {
    const uint4* va = reinterpret_cast<const uint4*>(pe + i0);
    const uint4* vb = reinterpret_cast<const uint4*>(pe + kHalfPe + i0);
    const uint4 a0 = __ldcg(va), a1 = __ldcg(va + 1), b0 = __ldcg(vb), b1 = __ldcg(vb + 1);
    ra[0] = a0.x; ra[1] = a0.y; ra[2] = a0.z; ra[3] = a0.w; ra[4] = a1.x; ra[5] = a1.y; ra[6] = a1.z; ra[7] = a1.w;
    rb[0] = b0.x; rb[1] = b0.y; rb[2] = b0.z; rb[3] = b0.w; rb[4] = b1.x; rb[5] = b1.y; rb[6] = b1.z; rb[7] = b1.w;
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      ra[k] = static_cast<uint32_t>(__ldcg(pe + i0 + 2 * k)) | (static_cast<uint32_t>(__ldcg(pe + i0 + 2 * k + 1)) << 16);
      rb[k] = static_cast<uint32_t>(__ldcg(pe + kHalfPe + i0 + 2 * k)) |
              (static_cast<uint32_t>(__ldcg(pe + kHalfPe + i0 + 2 * k + 1)) << 16);
    }
  }
  float c[16], s[16];
  bool on = false;
  if constexpr (ROPE) {
    on = pos >= 0 && pos < p.rope_rows;
    if (!on && h == 0 && (tid & 1) == 0) report(p.status, MLA_STATUS_POS_RANGE);
    if (on) {
      const float* tab = p.cos_sin + static_cast<int64_t>(pos) * kPe;
      if (p.tab_vec) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float4 cv = __ldg(reinterpret_cast<const float4*>(tab + i0) + k);
          const float4 sv = __ldg(reinterpret_cast<const float4*>(tab + kHalfPe + i0) + k);
          c[4 * k] = cv.x; c[4 * k + 1] = cv.y; c[4 * k + 2] = cv.z; c[4 * k + 3] = cv.w;
          s[4 * k] = sv.x; s[4 * k + 1] = sv.y; s[4 * k + 2] = sv.z; s[4 * k + 3] = sv.w;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          c[k] = __ldg(tab + i0 + k);
          s[k] = __ldg(tab + kHalfPe + i0 + k);
        }
      }
    }
  }
  float ya[16], yb[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const float a = (k & 1) ? bf16_hi(ra[k >> 1]) : bf16_lo(ra[k >> 1]);
    const float b = (k & 1) ? bf16_hi(rb[k >> 1]) : bf16_lo(rb[k >> 1]);
    ya[k] = a;
    yb[k] = b;
    if (ROPE && on) rope_pair(a, b, c[k], s[k], ya[k], yb[k]);
  }
  uint8_t* row = p.q_out + (static_cast<int64_t>(t) * p.H + h) * (QF8 ? kRow : 2 * kRow);
  if constexpr (QF8) {
    uint32_t wa[4], wb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      wa[j] = e4m3x2_of_f32<FAST>(ya[4 * j], ya[4 * j + 1], d) | (e4m3x2_of_f32<FAST>(ya[4 * j + 2], ya[4 * j + 3], d) << 16);
      wb[j] = e4m3x2_of_f32<FAST>(yb[4 * j], yb[4 * j + 1], d) | (e4m3x2_of_f32<FAST>(yb[4 * j + 2], yb[4 * j + 3], d) << 16);
    }
    *reinterpret_cast<uint4*>(row + kNope + i0) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    *reinterpret_cast<uint4*>(row + kNope + kHalfPe + i0) = make_uint4(wb[0], wb[1], wb[2], wb[3]);
  } else {
    uint32_t wa[8], wb[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      // an unrotated value keeps its bits (NaN payloads included)
      wa[j] = (ROPE && on) ? pack_bf16x2(ya[2 * j], ya[2 * j + 1]) : ra[j];
      wb[j] = (ROPE && on) ? pack_bf16x2(yb[2 * j], yb[2 * j + 1]) : rb[j];
    }
    uint4* da = reinterpret_cast<uint4*>(row + 2 * (kNope + i0));
    uint4* db = reinterpret_cast<uint4*>(row + 2 * (kNope + kHalfPe + i0));
    da[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    da[1] = make_uint4(wa[4], wa[5], wa[6], wa[7]);
    db[0] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
    db[1] = make_uint4(wb[4], wb[5], wb[6], wb[7]);
  }
}

__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag) {
  for (uint32_t i = 0; i < kWaitSpins; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    // the flag is read every 16 tries: shared-memory reads beside the tensor
    // cores' and the copy engine's traffic each cost about ten wavefronts
    if ((i & 15u) == 15u && *abort_flag != 0u) return false;
  }
  return false;
}

// barrier `id` over `n` threads, returning the AND of `pred` over them
__device__ __forceinline__ bool bar_and(int id, int n, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(n)
      : "memory");
  return out != 0u;
}

__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Contiguous-run tile order: (head, column half, token tile), token tile fastest.
struct TileCoord {
  int h, nt, m0;
};

__device__ __forceinline__ TileCoord tile_at(int idx, int mt) {
  TileCoord c;
  const int g = idx / mt;
  c.m0 = (idx - g * mt) * kM;
  c.h = g >> 1;
  c.nt = g & 1;
  return c;
}

struct Bars {
  uint64_t a_full[kStages], a_empty[kStages];
  uint64_t b_full, b_empty;
  uint64_t acc_full[2], acc_empty[2];
  uint64_t mma_done;
};

template <bool QF8, bool ROPE, bool FAST>
__device__ __forceinline__ void run(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmC,
                                    const Params& p, uint32_t sbase, const Bars& bars, uint32_t tmem,
                                    volatile uint32_t* abort_flag, const Divisor& d) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = (p.T + kM - 1) / kM;
  const int tiles = 2 * p.H * mt;
  const int per = tiles / static_cast<int>(gridDim.x);
  const int rem = tiles - per * static_cast<int>(gridDim.x);
  const int bx = static_cast<int>(blockIdx.x);
  const int combos = 2 * p.H;
  const int mains = p.per_combo * combos;
  const int mm = mt - p.tail;  // token tiles of the main part
  const bool main_cta = p.strided && bx < mains;
  const bool extra_cta = p.strided && bx >= mains;
  const int combo = bx % combos, j0 = bx / combos, step = p.per_combo;
  const int extras = static_cast<int>(gridDim.x) - mains;
  const int tail_tiles = p.tail * combos;
  const int e = bx - mains;
  const int lo = extra_cta ? static_cast<int>(static_cast<int64_t>(e) * tail_tiles / extras) : 0;
  const int hi = extra_cta ? static_cast<int>(static_cast<int64_t>(e + 1) * tail_tiles / extras) : 0;
  const int first = p.strided ? 0 : bx * per + (bx < rem ? bx : rem);
  const int count = main_cta ? (j0 < mm ? (mm - j0 + step - 1) / step : 0)
                    : extra_cta ? hi - lo
                                : per + (bx < rem ? 1 : 0);
  auto coord = [&](int i) -> TileCoord {
    if (main_cta) return TileCoord{combo >> 1, combo & 1, (j0 + i * step) * kM};
    if (extra_cta) {
      const int tau = lo + i;  // tail tiles in (head, half)-major order
      const int cb = tau / p.tail;
      return TileCoord{cb >> 1, cb & 1, (mm + tau - cb * p.tail) * kM};
    }
    return tile_at(first + i, mt);
  };
  const uint32_t sB = sbase;
  const uint32_t sA = sbase + kBBytes;
  const uint32_t sC = sA + kStages * kABytes;

  if (warp == kTmaWarp) {
    if (lane == 0) {
      bool waited = false;
      int group = -1, groups = 0, issued = 0;
      for (int i = 0; i < count && *abort_flag == 0u; ++i) {
        const TileCoord c = coord(i);
        const int g = c.h * 2 + c.nt;
        if (g != group) {
          if (groups > 0 && !wait_or_abort(smem_u32(&bars.b_empty), static_cast<uint32_t>(groups - 1) & 1u, abort_flag)) {
            *abort_flag = 1u;
            report(p.status, MLA_STATUS_TIMEOUT);
            break;
          }
          const uint32_t bf = smem_u32(&bars.b_full);
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bf), "r"(kBBytes) : "memory");
          tma_load_3d(sB, tmB, 0, c.nt * kN, c.h, bf);
          tma_load_3d(sB + kSlabB, tmB, 64, c.nt * kN, c.h, bf);
          group = g;
          ++groups;
        }
        const int st = i % kStages;
        const int use = i / kStages;
        if (use > 0 && !wait_or_abort(smem_u32(&bars.a_empty[st]), static_cast<uint32_t>(use - 1) & 1u, abort_flag)) {
          *abort_flag = 1u;
          report(p.status, MLA_STATUS_TIMEOUT);
          break;
        }
        if (!waited) {
          pdl_wait();  // the queries come from the upstream kernel
          waited = true;
        }
        const uint32_t af = smem_u32(&bars.a_full[st]);
        const uint32_t dst = sA + static_cast<uint32_t>(st) * kABytes;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(af), "r"(kABytes) : "memory");
        tma_load_3d(dst, tmA, 0, c.h, c.m0, af);
        tma_load_3d(dst + kSlabA, tmA, 64, c.h, c.m0, af);
        issued = i + 1;
      }
      // every copy issued has landed before the CTA may end
      for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
        (void)wait_phase(smem_u32(&bars.a_full[i % kStages]), static_cast<uint32_t>(i / kStages) & 1u);
      if (groups > 0) (void)wait_phase(smem_u32(&bars.b_full), static_cast<uint32_t>(groups - 1) & 1u);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      int group = -1, groups = 0;
      for (int i = 0; i < count && *abort_flag == 0u; ++i) {
        const TileCoord c = coord(i);
        const int g = c.h * 2 + c.nt;
        if (g != group) {
          if (!wait_or_abort(smem_u32(&bars.b_full), static_cast<uint32_t>(groups) & 1u, abort_flag)) {
            *abort_flag = 1u;
            report(p.status, MLA_STATUS_TIMEOUT);
            break;
          }
          group = g;
          ++groups;
        }
        const int st = i % kStages;
        const int b = i & 1;
        if (!wait_or_abort(smem_u32(&bars.a_full[st]), static_cast<uint32_t>(i / kStages) & 1u, abort_flag) ||
            (i >= 2 && !wait_or_abort(smem_u32(&bars.acc_empty[b]), static_cast<uint32_t>(i / 2 - 1) & 1u, abort_flag))) {
          *abort_flag = 1u;
          report(p.status, MLA_STATUS_TIMEOUT);
          break;
        }
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t a0 = sA + static_cast<uint32_t>(st) * kABytes;
        const uint32_t acc = tmem + static_cast<uint32_t>(b) * kN;
#pragma unroll
        for (int j = 0; j < kK / 16; ++j) {
          const uint32_t off = static_cast<uint32_t>(j & 3) * 32u;
          mma_bf16(acc, smem_desc_sw128(a0 + static_cast<uint32_t>(j >> 2) * kSlabA + off),
                   smem_desc_sw128(sB + static_cast<uint32_t>(j >> 2) * kSlabB + off), j > 0 ? 1u : 0u);
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&bars.a_empty[st]))
                     : "memory");
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                         smem_u32(&bars.acc_full[b]))
                     : "memory");
        bool last_of_group = (i + 1 == count);
        if (!last_of_group) {
          const TileCoord n = coord(i + 1);
          last_of_group = (n.h * 2 + n.nt) != g;
        }
        if (last_of_group)
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                           smem_u32(&bars.b_empty))
                       : "memory");
      }
      asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                       smem_u32(&bars.mma_done))
                   : "memory");
      (void)wait_phase(smem_u32(&bars.mma_done), 0u);
    }
  } else if (warp < kPeWarp0) {
    // epilogue: warp w reads TMEM lane quarter w mod 4, columns 128 hf .. 128 hf + 127
    const int ew = warp - kEpiWarp0;
    const int hf = ew >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const bool issuer = (ew & 3) == 0 && lane == 0;  // issues the bulk stores of its half
    constexpr int kSlabCols = QF8 ? 128 : 64;
    for (int i = 0; i < count; ++i) {
      const TileCoord c = coord(i);
      const int b = i & 1;
      // lane 0 polls for its warp; the barrier below orders the other lanes
      // after its wait, and the tcgen05 fence after the barrier orders the
      // accumulator reads after it
      bool ready = true;
      if (lane == 0)
        ready = wait_or_abort(smem_u32(&bars.acc_full[b]), static_cast<uint32_t>(i / 2) & 1u, abort_flag) &&
                *abort_flag == 0u;
      // e4m3 tiles (32 KB) alternate between the two halves of the 64 KB
      // staging area: wait only for the stores of two tiles back, which read
      // the half this tile writes; bf16 tiles fill it and wait for the last
      if (issuer) {
        if constexpr (QF8) {
          asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        } else {
          asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        }
      }
      if (!bar_and(1, 32 * kEpiWarps, ready)) {
        if (lane == 0 && ew == 0) {
          *abort_flag = 1u;
          report(p.status, MLA_STATUS_TIMEOUT);
        }
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t acc = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(b) * kN;
      const uint32_t sCb = QF8 ? sC + static_cast<uint32_t>(b) * 2u * kSlabC : sC;
#pragma unroll 1
      for (int col = hf * 128; col < hf * 128 + 128; col += 32) {
        uint32_t v[32];
        tmem_ld32(acc + static_cast<uint32_t>(col), v);
        stage_chunk<QF8, FAST>(sCb, r, col, v, d);
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bars.acc_empty[b])) : "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      bar_sync(2 + hf, 128);
      if (issuer) {
#pragma unroll
        for (int sl = hf * (128 / kSlabCols); sl < (hf + 1) * (128 / kSlabCols); ++sl)
          tma_store_3d(tmC, sCb + static_cast<uint32_t>(sl) * kSlabC, c.nt * kN + sl * kSlabCols, c.h, c.m0);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      }
    }
    if (issuer) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  } else {
    // rotary warps: the 64 pe values of every head of this CTA's share of
    // the tokens (independent of its tiles), item (t, h, half) per thread,
    // consecutive threads on consecutive heads of one token
    const int slot = static_cast<int>(threadIdx.x) - 32 * kPeWarp0;
    const int64_t tb0 = static_cast<int64_t>(p.T) * bx / static_cast<int>(gridDim.x);
    const int64_t tb1 = static_cast<int64_t>(p.T) * (bx + 1) / static_cast<int>(gridDim.x);
    const int64_t per_token = 2 * static_cast<int64_t>(p.H);
    const int64_t items = (tb1 - tb0) * per_token;
    pdl_wait();  // q_pe comes from the upstream kernel
    for (int64_t it = slot; it < items; it += 32 * kPeWarps) {
      const int64_t tt = it / per_token;
      const int rem = static_cast<int>(it - tt * per_token);
      pe_part<QF8, ROPE, FAST>(p, static_cast<int>(tb0 + tt), 0, rem >> 1, rem & 1, d);
    }
  }
}

template <bool QF8, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
    absorb_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const __grid_constant__ CUtensorMap tmC, const Params p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) Bars bars;
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t abort_flag;
  const int warp = threadIdx.x >> 5;
  const uint32_t sbase = (smem_u32(dsmem) + 1023u) & ~1023u;
  float q_scale = 1.0f;
  if constexpr (QF8) q_scale = __ldg(p.q_scale);

  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 0) {
    abort_flag = 0u;
    for (int st = 0; st < kStages; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.a_full[st])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.a_empty[st])) : "memory");
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.b_full)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.b_empty)) : "memory");
    for (int b = 0; b < 2; ++b) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.acc_full[b])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(&bars.acc_empty[b])), "r"(kEpiWarps) : "memory");
    }
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&bars.mma_done)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_slot;

  Divisor d{};
  d.fast = true;
  if constexpr (QF8) d = make_divisor(q_scale);
  if (d.fast) {
    run<QF8, ROPE, true>(&tmA, &tmB, &tmC, p, sbase, bars, tmem, &abort_flag, d);
  } else {
    run<QF8, ROPE, false>(&tmA, &tmB, &tmC, p, sbase, bars, tmem, &abort_flag, d);
  }

  // every MMA has completed (the MMA warp waited for its final commit) and
  // every copy has landed (the TMA warp drained them): free the TMEM
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
  pdl_trigger();
}

template <bool QF8, bool ROPE>
const void* kernel_for() {
  return reinterpret_cast<const void*>(&absorb_kernel<QF8, ROPE>);
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess) {
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    } else {
      (void)cudaGetLastError();
    }
  }
  return fn;
}

// Whether the kernel for flag bits k has its shared-memory opt-in on device
// `dev` (cudaFuncSetAttribute applies per device).
std::atomic<bool> g_smem_ready[kMaxDevices][4];

}  // namespace absorb
}  // namespace mla

extern "C" {

mla_status mla_absorb_launch(const void* q_nope_c, int64_t qc_st, int64_t qc_sh, const void* w_uk, const void* q_pe,
                             int64_t qp_st, int64_t qp_sh, const int32_t* positions, const float* cos_sin,
                             int64_t rope_rows, const float* q_scale, int64_t T, int64_t H, uint32_t flags,
                             void* q_out, int32_t* status, mla_stream_t stream) {
  using namespace mla::absorb;
  if ((flags & ~(MLA_FLAG_ROPE | MLA_FLAG_Q_FP8 | MLA_FLAG_PDL)) != 0) return MLA_ERR_UNSUPPORTED;
  // T * H < 2^31 - 128: every token, tile and row index of the kernel (T rounded up to a whole tile
  // included) stays in 32 bits
  if (T < 0 || H < 1 || H > 65535 || T > (static_cast<int64_t>(INT_MAX) - kM) / H) return MLA_ERR_INVALID_ARG;
  const bool rope = (flags & MLA_FLAG_ROPE) != 0;
  const bool qf8 = (flags & MLA_FLAG_Q_FP8) != 0;
  if (rope && (rope_rows < 1 || rope_rows > (INT64_C(1) << 40))) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (q_nope_c == nullptr || w_uk == nullptr || q_pe == nullptr || q_out == nullptr) return MLA_ERR_INVALID_ARG;
  if (rope && (positions == nullptr || cos_sin == nullptr)) return MLA_ERR_INVALID_ARG;
  if (qf8 && q_scale == nullptr) return MLA_ERR_INVALID_ARG;
  if (qc_st < 0 || qc_sh < 0 || qp_st < 0 || qp_sh < 0) return MLA_ERR_INVALID_ARG;
  auto aligned = [](const void* ptr, uintptr_t n) { return (reinterpret_cast<uintptr_t>(ptr) % n) == 0; };
  if (!aligned(q_nope_c, 16) || !aligned(w_uk, 16) || !aligned(q_out, 16) || !aligned(q_pe, 2)) return MLA_ERR_ALIGNMENT;
  if ((T > 1 && (qc_st % 8) != 0) || (H > 1 && (qc_sh % 8) != 0)) return MLA_ERR_ALIGNMENT;
  if ((rope && (!aligned(positions, 4) || !aligned(cos_sin, 4))) || (qf8 && !aligned(q_scale, 4)) ||
      (status != nullptr && !aligned(status, 4)))
    return MLA_ERR_ALIGNMENT;

  int dev = 0;
  int32_t sms = 0;
  const mla_status ds = mla::current_device(&dev, &sms);
  if (ds != MLA_OK) return ds;
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return mla::cuda_failure(cudaErrorNotSupported);

  // A: q_nope_c as (k, h, t), box (64, 1, 128); a size-1 dimension gets any
  // legal stride (it is never stepped over)
  CUtensorMap tmA, tmB;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kK), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(H > 1 ? qc_sh : kK) * 2,
                                   static_cast<cuuint64_t>(T > 1 ? qc_st : kK * H) * 2};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kM)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q_nope_c), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_INVALID_ARG;
  }
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kK), static_cast<cuuint64_t>(kNope),
                                static_cast<cuuint64_t>(H)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kK) * 2, static_cast<cuuint64_t>(kNope * kK) * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kN), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w_uk), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_INVALID_ARG;
  }

  // C: q_out as (column, h, t), box (one 128-byte column slab, 1, 128), written
  // from the 128-byte swizzled staging tile; rows past T are not written
  CUtensorMap tmC;
  {
    const cuuint64_t esz = qf8 ? 1 : 2;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(kRow), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(kRow) * esz, static_cast<cuuint64_t>(kRow * H) * esz};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), 1, static_cast<cuuint32_t>(kM)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&tmC, qf8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q_out, dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return MLA_ERR_INVALID_ARG;
  }

  Params prm;
  prm.q_pe = static_cast<const uint16_t*>(q_pe);
  prm.qp_st = qp_st;
  prm.qp_sh = qp_sh;
  prm.positions = positions;
  prm.cos_sin = cos_sin;
  prm.rope_rows = rope ? rope_rows : 0;
  prm.q_scale = q_scale;
  prm.T = static_cast<int32_t>(T);
  prm.H = static_cast<int32_t>(H);
  prm.q_out = static_cast<uint8_t*>(q_out);
  prm.status = status;
  prm.pe_vec = aligned(q_pe, 16) && (T == 1 || qp_st % 8 == 0) && (H == 1 || qp_sh % 8 == 0);
  prm.tab_vec = rope && aligned(cos_sin, 16);
  prm.strided = (2 * H <= sms) ? 1 : 0;
  prm.per_combo = prm.strided ? static_cast<int32_t>(sms / (2 * H)) : 1;
  prm.tail = 0;
  if (prm.strided) {
    // tail tiles per (head, half) that balance the main CTAs, (mt - tail) / R
    // tiles each, against the E extras, tail * 2H / E each: the balance point
    // mt E / (E + R 2H), and its neighbours for the rounding
    const int64_t mt = (T + kM - 1) / kM, C = 2 * H, R = prm.per_combo, E = sms - R * C;
    int64_t best = 0, best_span = (mt + R - 1) / R;
    if (E > 0) {
      const int64_t t0 = mt * E / (E + R * C);
      for (int64_t tl = t0 > 2 ? t0 - 2 : 0; tl <= t0 + 3 && tl <= mt; ++tl) {
        const int64_t main_span = (mt - tl + R - 1) / R, extra_span = (tl * C + E - 1) / E;
        const int64_t span = main_span > extra_span ? main_span : extra_span;
        if (span < best_span) {
          best_span = span;
          best = tl;
        }
      }
    }
    prm.tail = static_cast<int32_t>(best);
  }

  const int k = (qf8 ? 2 : 0) | (rope ? 1 : 0);
  static const void* const kernels[4] = {kernel_for<false, false>(), kernel_for<false, true>(),
                                         kernel_for<true, false>(), kernel_for<true, true>()};
  const void* fn = kernels[k];
  if (!g_smem_ready[dev][k].load(std::memory_order_acquire)) {
    // idempotent: two threads racing here both set the same attribute
    const cudaError_t e =
        cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return mla::cuda_failure(e);
    g_smem_ready[dev][k].store(true, std::memory_order_release);
  }

  cudaLaunchConfig_t cfg = {};
  const int64_t tiles = 2 * H * ((T + kM - 1) / kM);
  int64_t grid = tiles < sms ? tiles : sms;
  if (prm.strided) grid = prm.tail > 0 ? sms : prm.per_combo * 2 * H;
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = reinterpret_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  if (flags & MLA_FLAG_PDL) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  void* args[] = {&tmA, &tmB, &tmC, &prm};
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return mla::cuda_failure(e);
  return MLA_OK;
}

}  // extern "C"
