// mla_absorb.cu -- latent query rows straight from the absorption product, on
// the tcgen05 tensor cores (contract in mla_absorb.h).
//
// One CTA of four warps computes a 128-token x 256-column tile of one head:
//   * the A tile (q_nope_c: 128 tokens x 128) and the B tile (w_uk: 256 latent
//     rows x 128) arrive by TMA with the 128-byte swizzle, as two 64-wide
//     column slabs each, on one mbarrier; the weights are requested before
//     the kernel waits for the upstream grid, the query after;
//   * one thread issues eight M=128, N=256, K=16 tcgen05.mma (bf16 in, fp32
//     accumulate) into 256 TMEM columns and commits them to a second mbarrier;
//   * each warp reads its 32 TMEM lanes (tokens) back with tcgen05.ld, 32
//     columns at a time, and writes them encoded (bf16, or e4m3 of x / scale)
//     straight into q_out's row layout;
//   * the CTAs of the second column tile also rotate and write the 64 pe
//     values of their 128 tokens, one RoPE pair per lane, while the tensor
//     cores run.
// The weights of a head are 128 KB and stay in L2 across tiles; the two column
// tiles of one token tile are adjacent in the grid so the A tile is read from
// HBM once.  Every wait is bounded: on timeout the kernel sets a status bit,
// waits (bounded) for what it issued, frees its TMEM and returns.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>

#include "latent_math.cuh"
#include "mla_absorb.h"

namespace mla {
namespace absorb {

constexpr int kM = 128;          // tokens per tile (UMMA M)
constexpr int kN = 256;          // latent columns per tile (UMMA N)
constexpr int kK = 128;          // contraction (nope head dim before absorption)
constexpr int kNope = 512;
constexpr int kPe = 64;
constexpr int kHalfPe = 32;
constexpr int kRow = 576;
constexpr int kThreads = 128;
constexpr uint32_t kSlabA = kM * 64 * 2;     // one 64-wide column slab of A: 16 KB
constexpr uint32_t kSlabB = kN * 64 * 2;     // one 64-wide column slab of B: 32 KB
constexpr uint32_t kTileBytes = 2 * kSlabA + 2 * kSlabB;  // 96 KB
constexpr uint32_t kSmemBytes = kTileBytes + 1024;        // + room to align to 1024
constexpr uint32_t kTmemCols = 256;
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
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 32 accumulator values (columns c..c+31 of one token row) -> q_out.
template <bool QF8, bool FAST>
__device__ __forceinline__ void store_chunk(uint8_t* row, int col, const uint32_t (&v)[32], const Divisor& d) {
  if constexpr (QF8) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = e4m3x2_of_f32<FAST>(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), d);
      const uint32_t hi = e4m3x2_of_f32<FAST>(__uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]), d);
      w[i] = lo | (hi << 16);
    }
    uint4* dst = reinterpret_cast<uint4*>(row + col);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    uint4* dst = reinterpret_cast<uint4*>(row + 2 * col);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

// The 64 rotary values of tokens m0..m0+127 of head h: warp w takes rows
// w, w+4, ...; lane i the pair (i, i+32).
template <bool QF8, bool ROPE, bool FAST>
__device__ __forceinline__ void pe_rows(const Params& p, int m0, int h, const Divisor& d) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  for (int r = warp; r < kM; r += kThreads / 32) {
    const int t = m0 + r;
    if (t >= p.T) break;
    float c = 1.0f, s = 0.0f;
    bool on = false;
    if constexpr (ROPE) {
      const int64_t pos = __ldg(p.positions + t);
      if (pos >= 0 && pos < p.rope_rows) {
        const float* tab = p.cos_sin + pos * kPe;
        c = __ldg(tab + lane);
        s = __ldg(tab + kHalfPe + lane);
        on = true;
      } else if (lane == 0 && h == 0) {
        report(p.status, MLA_STATUS_POS_RANGE);
      }
    }
    const uint16_t* pe = p.q_pe + static_cast<int64_t>(t) * p.qp_st + static_cast<int64_t>(h) * p.qp_sh;
    const uint32_t raw = static_cast<uint32_t>(__ldcg(pe + lane)) | (static_cast<uint32_t>(__ldcg(pe + kHalfPe + lane)) << 16);
    float a = bf16_lo(raw), b = bf16_hi(raw);
    bool rotated = false;
    if (ROPE && on) {
      float ya, yb;
      rope_pair(a, b, c, s, ya, yb);
      a = ya;
      b = yb;
      rotated = true;
    }
    uint8_t* row = p.q_out + (static_cast<int64_t>(t) * p.H + h) * (QF8 ? kRow : 2 * kRow);
    if constexpr (QF8) {
      const uint32_t e = e4m3x2_of_f32<FAST>(a, b, d);
      row[kNope + lane] = static_cast<uint8_t>(e & 0xffu);
      row[kNope + kHalfPe + lane] = static_cast<uint8_t>((e >> 8) & 0xffu);
    } else {
      const uint32_t o = rotated ? pack_bf16x2(a, b) : raw;
      uint16_t* r16 = reinterpret_cast<uint16_t*>(row);
      r16[kNope + lane] = static_cast<uint16_t>(o & 0xffffu);
      r16[kNope + kHalfPe + lane] = static_cast<uint16_t>(o >> 16);
    }
  }
}

template <bool QF8, bool ROPE, bool FAST>
__device__ __forceinline__ void tile(const CUtensorMap* tmA, const CUtensorMap* tmB, const Params& p,
                                     uint32_t sbase, uint32_t bar_tma, uint32_t bar_mma, uint32_t tmem,
                                     volatile uint32_t* fail, const Divisor& d) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m0 = static_cast<int>(blockIdx.x >> 1) * kM;
  const int nt = static_cast<int>(blockIdx.x & 1u);
  const int n0 = nt * kN;
  const int h = static_cast<int>(blockIdx.y);
  const uint32_t sA = sbase;                  // two 16 KB slabs: k 0..63, 64..127
  const uint32_t sB = sbase + 2 * kSlabA;     // two 32 KB slabs

  if (threadIdx.x == 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_tma), "r"(kTileBytes)
                 : "memory");
    // weights do not depend on the upstream kernel
    tma_load_3d(sB, tmB, 0, n0, h, bar_tma);
    tma_load_3d(sB + kSlabB, tmB, 64, n0, h, bar_tma);
    pdl_wait();
    tma_load_3d(sA, tmA, 0, h, m0, bar_tma);
    tma_load_3d(sA + kSlabA, tmA, 64, h, m0, bar_tma);
    if (wait_phase(bar_tma, 0)) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int j = 0; j < kK / 16; ++j) {
        // K step j: slab j/4, 32 bytes (16 bf16) further per step inside the 128-byte row
        const uint32_t off = static_cast<uint32_t>(j & 3) * 32u;
        const uint64_t a = smem_desc_sw128(sA + static_cast<uint32_t>(j >> 2) * kSlabA + off);
        const uint64_t b = smem_desc_sw128(sB + static_cast<uint32_t>(j >> 2) * kSlabB + off);
        mma_bf16(tmem, a, b, j > 0 ? 1u : 0u);
      }
    } else {
      *fail = 1u;
      report(p.status, MLA_STATUS_TIMEOUT);
      (void)wait_phase(bar_tma, 0);  // the copies may still land: give them one more bounded wait
    }
    // arrives once every MMA issued above has completed (at once if none was)
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_mma)
                 : "memory");
  }

  if (nt == 1) {
    pdl_wait();  // q_pe comes from the upstream kernel
    pe_rows<QF8, ROPE, FAST>(p, m0, h, d);
  }

  // warp-uniform: tcgen05.ld below is a whole-warp instruction
  const bool ok = __all_sync(0xffffffffu, wait_phase(bar_mma, 0));
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (!ok) {
    if (lane == 0) report(p.status, MLA_STATUS_TIMEOUT);
    return;
  }
  if (__any_sync(0xffffffffu, *fail != 0u)) return;
  const int r = warp * 32 + lane;  // TMEM lane = accumulator row = token m0 + r
  const int t = m0 + r;
  uint8_t* row = p.q_out + (static_cast<int64_t>(t) * p.H + h) * (QF8 ? kRow : 2 * kRow);
#pragma unroll 1
  for (int c = 0; c < kN; c += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c), v);
    if (t < p.T) store_chunk<QF8, FAST>(row, n0 + c, v, d);
  }
}

template <bool QF8, bool ROPE>
__global__ void __launch_bounds__(kThreads, 1)
    absorb_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const Params p) {
  extern __shared__ uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ uint32_t tmem_slot;
  __shared__ uint32_t fail;
  const int warp = threadIdx.x >> 5;
  const uint32_t sbase = (smem_u32(dsmem) + 1023u) & ~1023u;
  const uint32_t bar_tma = smem_u32(&bars[0]);
  const uint32_t bar_mma = smem_u32(&bars[1]);

  Divisor d{};
  d.fast = true;
  if constexpr (QF8) d = make_divisor(__ldg(p.q_scale));

  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 0) {
    fail = 0u;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_tma) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_slot;

  if (d.fast) {
    tile<QF8, ROPE, true>(&tmA, &tmB, p, sbase, bar_tma, bar_mma, tmem, &fail, d);
  } else {
    tile<QF8, ROPE, false>(&tmA, &tmB, p, sbase, bar_tma, bar_mma, tmem, &fail, d);
  }

  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 1) {
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

}  // namespace absorb
}  // namespace mla

extern "C" {

mla_status mla_absorb_launch(const void* q_nope_c, int64_t qc_st, int64_t qc_sh, const void* w_uk, const void* q_pe,
                             int64_t qp_st, int64_t qp_sh, const int32_t* positions, const float* cos_sin,
                             int64_t rope_rows, const float* q_scale, int64_t T, int64_t H, uint32_t flags,
                             void* q_out, int32_t* status, mla_stream_t stream) {
  using namespace mla::absorb;
  if ((flags & ~(MLA_FLAG_ROPE | MLA_FLAG_Q_FP8 | MLA_FLAG_PDL)) != 0) return MLA_ERR_UNSUPPORTED;
  if (T < 0 || H < 1 || H > 65535 || T > static_cast<int64_t>(INT_MAX) / H) return MLA_ERR_INVALID_ARG;
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

  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (encode == nullptr) return MLA_ERR_CUDA;

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

  const int k = (qf8 ? 2 : 0) | (rope ? 1 : 0);
  static const void* const kernels[4] = {kernel_for<false, false>(), kernel_for<false, true>(),
                                         kernel_for<true, false>(), kernel_for<true, true>()};
  static bool smem_set[4] = {false, false, false, false};
  const void* fn = kernels[k];
  if (!smem_set[k]) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes)) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return MLA_ERR_CUDA;
    }
    smem_set[k] = true;
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(((T + kM - 1) / kM) * 2), static_cast<unsigned>(H), 1);
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
  void* args[] = {&tmA, &tmB, &prm};
  const cudaError_t e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MLA_ERR_CUDA;
  }
  return MLA_OK;
}

}  // extern "C"
