// mla_harness.cu -- the kernels that sit beside the epilogue: synthetic
// producers (copy-only, or streaming a weight buffer first), empty kernels for
// the launch floors, a synthetic consumer, and two device checks of the e4m3
// quotient (declarations and contracts in mla_harness.h).

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "latent_math.cuh"
#include "mla_harness.h"
#include "mla_runtime.h"

namespace mla {
namespace harness {

// One warp per (token, head) row: 1024 bytes of nope (two 16-byte chunks per
// lane) and 128 bytes of pe (lanes 0..7), grid-stride.
// With `weights`: first every thread reads its grid-stride share of the
// weights (16-byte words) and each block XORs what it read into *sink.
__global__ void __launch_bounds__(256) produce_kernel(const uint4* __restrict__ src_nope,
                                                      const uint4* __restrict__ src_pe,
                                                      uint16_t* q_nope, int64_t qn_st, int64_t qn_sh,
                                                      uint16_t* q_pe, int64_t qp_st, int64_t qp_sh,
                                                      int64_t T, int64_t H, const uint4* __restrict__ weights,
                                                      int64_t weight_words, uint32_t* sink) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (weight_words > 0) {
    const int64_t threads = static_cast<int64_t>(gridDim.x) * blockDim.x;
    uint32_t acc = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < weight_words; i += threads) {
      const uint4 w = __ldcs(weights + i);
      acc ^= w.x ^ w.y ^ w.z ^ w.w;
    }
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0 && acc != 0u) atomicXor(sink, acc);
  }
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t rows = T * H;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const int64_t t = r / H;
    const int64_t h = r - t * H;
    const uint4 a = src_nope[r * 64 + lane];
    const uint4 b = src_nope[r * 64 + 32 + lane];
    uint4 p = make_uint4(0, 0, 0, 0);
    if (lane < 8) p = src_pe[r * 8 + lane];
    uint4* dn = reinterpret_cast<uint4*>(q_nope + t * qn_st + h * qn_sh);
    dn[lane] = a;
    dn[32 + lane] = b;
    if (lane < 8) reinterpret_cast<uint4*>(q_pe + t * qp_st + h * qp_sh)[lane] = p;
  }
}

__global__ void empty_kernel() {}

__global__ void empty_wait_kernel() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Quotient of one fp32 through the epilogue's e4m3 path (the pair function
// with the second lane unused), returned as the fp32 quotient it encodes.
__device__ __forceinline__ float epilogue_quotient(float x, const Divisor& d) {
  if (!d.fast) return __fdiv_rn(x, d.s);
  float q, unused;
  quotient_pair_neg(neg_clamp(x, d), neg_clamp(0.0f, d), d, q, unused);
  return q;
}

__global__ void __launch_bounds__(256) div_check_kernel(float scale, uint64_t first, uint64_t count,
                                                        unsigned long long* result) {
  const Divisor d = make_divisor(scale);
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  unsigned long long bad_q = 0, bad_b = 0, lowest = ~0ull;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count; i += stride) {
    const uint64_t p = first + i;
    const uint32_t w = static_cast<uint32_t>(p);
    const float x = __uint_as_float(w);
    const float q = epilogue_quotient(x, d);
    const float ref = __fdiv_rn(x, scale);
    const bool same_q = (__float_as_uint(q) == __float_as_uint(ref)) || (isnan(q) && isnan(ref));
    // fp32 path (rotated values): the byte the epilogue stores vs the byte of the IEEE quotient
    const uint32_t bq = (d.fast ? e4m3x2_of_f32<true>(x, 0.0f, d) : e4m3x2_of_f32<false>(x, 0.0f, d)) & 0xffu;
    const uint32_t br = pack_e4m3x2(ref, 0.0f) & 0xffu;
    // bf16x2 path (unrotated inputs): the two halves of the pattern as bf16
    const uint32_t bb = d.fast ? e4m3x2_of_bf16x2<true>(w, d) : e4m3x2_of_bf16x2<false>(w, d);
    const uint32_t bbr = pack_e4m3x2(__fdiv_rn(bf16_lo(w), scale), __fdiv_rn(bf16_hi(w), scale));
    // quotient bits are compared where they decide an e4m3 byte and the
    // epilogue computes the IEEE quotient: |x| >= 2^-100 (below, the residual may
    // underflow; |x / scale| <= 2^-36 rounds to a signed zero) and
    // |x / scale| < 448 (above, the input is clamped; the byte saturates)
    if (!same_q && fabsf(x) >= 0x1p-100f && !(fabsf(ref) >= 448.0f)) {
      ++bad_q;
      if (p < lowest) lowest = p;
    }
    if (bq != br || bb != bbr) {
      ++bad_b;
      if (p < lowest) lowest = p;
    }
  }
  if (bad_q) atomicAdd(result + 0, bad_q);
  if (bad_b) atomicAdd(result + 1, bad_b);
  if (lowest != ~0ull) atomicMin(result + 2, lowest);
}

// Every bf16 value through the epilogue's e4m3 path against the byte of the
// IEEE quotient, for scale bit patterns [first, first + count).  Item i is
// scale first + i / 8 and bf16 pairs (2k, 2k + 1) for k in one eighth of
// [0, 32768).
__global__ void __launch_bounds__(256) bf16_scale_check_kernel(uint32_t first, uint32_t count,
                                                               unsigned long long* result) {
  constexpr uint32_t kParts = 8, kPairs = 32768 / kParts;
  const uint64_t items = static_cast<uint64_t>(count) * kParts;
  const uint64_t stride = static_cast<uint64_t>(gridDim.x) * blockDim.x;
  unsigned long long bad = 0, lowest = ~0ull;
  for (uint64_t i = static_cast<uint64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < items; i += stride) {
    const uint32_t bits = first + static_cast<uint32_t>(i / kParts);
    const float scale = __uint_as_float(bits);
    const Divisor d = make_divisor(scale);
    const uint32_t k0 = static_cast<uint32_t>(i % kParts) * kPairs;
    uint32_t n = 0;
    for (uint32_t k = k0; k < k0 + kPairs; ++k) {
      const uint32_t w = ((2u * k + 1u) << 16) | (2u * k);
      const uint32_t got = d.fast ? e4m3x2_of_bf16x2<true>(w, d) : e4m3x2_of_bf16x2<false>(w, d);
      const uint32_t ref = pack_e4m3x2(__fdiv_rn(bf16_lo(w), scale), __fdiv_rn(bf16_hi(w), scale));
      n += ((got ^ ref) & 0xffu) != 0u;
      n += ((got ^ ref) & 0xff00u) != 0u;
    }
    if (n != 0u) {
      bad += n;
      if (bits < lowest) lowest = bits;
    }
  }
  if (bad) atomicAdd(result + 0, bad);
  if (lowest != ~0ull) atomicMin(result + 1, lowest);
}

// e4m3 byte -> fp32 (exact: every e4m3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint8_t b) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(b)));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xffffu)));
}

template <bool QF8, bool KVF8>
__global__ void __launch_bounds__(256) consume_kernel(const uint8_t* q_out, const uint8_t* cache,
                                                      const int64_t* slots, int64_t T, int64_t H,
                                                      int64_t cache_rows, float* scores) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  // slot_mapping is not written by the epilogue: read it before waiting
  int64_t slot = first < T * H ? __ldg(slots + first / H) : 0;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int64_t r = first; r < T * H; r += warps) {
    if (r != first) slot = __ldg(slots + r / H);
    if (slot < 0 || slot >= cache_rows) {
      if (lane == 0) scores[r] = __int_as_float(0x7fc00000);
      continue;
    }
    const uint8_t* q = q_out + r * (QF8 ? 576 : 1152);
    const uint8_t* k = cache + slot * (KVF8 ? 576 : 1152);
    float acc = 0.0f;
    for (int i = lane; i < 576; i += 32) {
      const float qv = QF8 ? e4m3_to_f32(__ldcg(q + i)) : bf16_bits(__ldcg(reinterpret_cast<const uint16_t*>(q) + i));
      const float kv = KVF8 ? e4m3_to_f32(__ldcg(k + i)) : bf16_bits(__ldcg(reinterpret_cast<const uint16_t*>(k) + i));
      acc = __fmaf_rn(qv, kv, acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) scores[r] = acc;
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mla_status finish(cudaError_t e) { return e == cudaSuccess ? MLA_OK : cuda_failure(e); }

mla_status launch(const void* fn, dim3 grid, dim3 block, bool pdl, cudaStream_t stream, void** args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return finish(cudaLaunchKernelExC(&cfg, fn, args));
}

mla_status produce(const void* src_nope, const void* src_pe, void* q_nope, int64_t q_nope_stride_t,
                   int64_t q_nope_stride_h, void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
                   const void* weights, int64_t weight_bytes, uint32_t* sink, int64_t T, int64_t H, uint32_t flags,
                   mla_stream_t stream) {
  if ((flags & ~MLA_FLAG_PDL) != 0) return MLA_ERR_UNSUPPORTED;
  if (T < 0 || H < 1 || T > (INT64_C(1) << 31) / H || weight_bytes < 0) return MLA_ERR_INVALID_ARG;
  if (weight_bytes > 0 && (weights == nullptr || sink == nullptr)) return MLA_ERR_INVALID_ARG;
  if (weight_bytes > 0 && (!aligned16(weights) || (weight_bytes % 16) != 0 ||
                           (reinterpret_cast<uintptr_t>(sink) & 3u) != 0))
    return MLA_ERR_ALIGNMENT;
  if (T == 0 && weight_bytes == 0) return MLA_OK;
  if (T > 0) {
    if (!src_nope || !src_pe || !q_nope || !q_pe) return MLA_ERR_INVALID_ARG;
    if (q_nope_stride_t < 0 || q_nope_stride_h < 0 || q_pe_stride_t < 0 || q_pe_stride_h < 0)
      return MLA_ERR_INVALID_ARG;
    if (!aligned16(src_nope) || !aligned16(src_pe) || !aligned16(q_nope) || !aligned16(q_pe) ||
        (q_nope_stride_t % 8) || (q_nope_stride_h % 8) || (q_pe_stride_t % 8) || (q_pe_stride_h % 8))
      return MLA_ERR_ALIGNMENT;
  }
  int32_t sms = 0;
  const mla_status s = mla::current_device(nullptr, &sms);
  if (s != MLA_OK) return s;
  const int64_t rows = T * H;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  if (weight_bytes > 0 && blocks < static_cast<int64_t>(sms) * 4) blocks = static_cast<int64_t>(sms) * 4;
  const uint4* sn = static_cast<const uint4*>(src_nope);
  const uint4* sp = static_cast<const uint4*>(src_pe);
  uint16_t* qn = static_cast<uint16_t*>(q_nope);
  uint16_t* qp = static_cast<uint16_t*>(q_pe);
  const uint4* wt = static_cast<const uint4*>(weights);
  int64_t words = weight_bytes / 16;
  void* args[] = {&sn, &sp, &qn, &q_nope_stride_t, &q_nope_stride_h, &qp, &q_pe_stride_t, &q_pe_stride_h,
                  &T, &H, &wt, &words, &sink};
  return launch(reinterpret_cast<const void*>(&produce_kernel), dim3(static_cast<unsigned>(blocks)), dim3(256),
                (flags & MLA_FLAG_PDL) != 0, reinterpret_cast<cudaStream_t>(stream), args);
}

}  // namespace harness
}  // namespace mla

extern "C" {


mla_status mla_harness_produce(const void* src_nope, const void* src_pe, void* q_nope, int64_t q_nope_stride_t,
                               int64_t q_nope_stride_h, void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
                               int64_t T, int64_t H, uint32_t flags, mla_stream_t stream) {
  return mla::harness::produce(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h, q_pe, q_pe_stride_t,
                               q_pe_stride_h, nullptr, 0, nullptr, T, H, flags, stream);
}

mla_status mla_harness_produce_after_weights(const void* src_nope, const void* src_pe, void* q_nope,
                                             int64_t q_nope_stride_t, int64_t q_nope_stride_h, void* q_pe,
                                             int64_t q_pe_stride_t, int64_t q_pe_stride_h, const void* weights,
                                             int64_t weight_bytes, uint32_t* sink, int64_t T, int64_t H,
                                             uint32_t flags, mla_stream_t stream) {
  return mla::harness::produce(src_nope, src_pe, q_nope, q_nope_stride_t, q_nope_stride_h, q_pe, q_pe_stride_t,
                               q_pe_stride_h, weights, weight_bytes, sink, T, H, flags, stream);
}

mla_status mla_harness_empty(int64_t blocks, int32_t threads, uint32_t flags, mla_stream_t stream) {
  using namespace mla::harness;
  if ((flags & ~(MLA_FLAG_PDL | MLA_HARNESS_EMPTY_WAIT)) != 0) return MLA_ERR_UNSUPPORTED;
  if (blocks < 1 || blocks > INT32_MAX || threads < 1 || threads > 1024) return MLA_ERR_INVALID_ARG;
  const void* fn = (flags & MLA_HARNESS_EMPTY_WAIT) ? reinterpret_cast<const void*>(&empty_wait_kernel)
                                                    : reinterpret_cast<const void*>(&empty_kernel);
  return launch(fn, dim3(static_cast<unsigned>(blocks)),
                dim3(static_cast<unsigned>(threads)), (flags & MLA_FLAG_PDL) != 0,
                reinterpret_cast<cudaStream_t>(stream), nullptr);
}

mla_status mla_harness_div_check(float scale, uint64_t first, uint64_t count, unsigned long long* result,
                                 mla_stream_t stream) {
  using namespace mla::harness;
  if (result == nullptr || (reinterpret_cast<uintptr_t>(result) & 7u) != 0) return MLA_ERR_INVALID_ARG;
  if (first > (UINT64_C(1) << 32) || count > (UINT64_C(1) << 32) - first) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(result, 0, 2 * sizeof(unsigned long long), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(result + 2, 0xff, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return finish(e);
  if (count == 0) return MLA_OK;
  int32_t sms = 0;
  const mla_status st = mla::current_device(nullptr, &sms);
  if (st != MLA_OK) return st;
  void* args[] = {&scale, &first, &count, &result};
  return launch(reinterpret_cast<const void*>(&div_check_kernel), dim3(static_cast<unsigned>(sms) * 16), dim3(256),
                false, s, args);
}

mla_status mla_harness_bf16_scale_check(uint32_t first, uint32_t count, unsigned long long* result,
                                        mla_stream_t stream) {
  using namespace mla::harness;
  if (result == nullptr || (reinterpret_cast<uintptr_t>(result) & 7u) != 0) return MLA_ERR_INVALID_ARG;
  if (static_cast<uint64_t>(first) + count > (UINT64_C(1) << 32)) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(result, 0, sizeof(unsigned long long), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(result + 1, 0xff, sizeof(unsigned long long), s);
  if (e != cudaSuccess) return finish(e);
  if (count == 0) return MLA_OK;
  int32_t sms = 0;
  const mla_status st = mla::current_device(nullptr, &sms);
  if (st != MLA_OK) return st;
  void* args[] = {&first, &count, &result};
  return launch(reinterpret_cast<const void*>(&bf16_scale_check_kernel), dim3(static_cast<unsigned>(sms) * 16),
                dim3(256), false, s, args);
}

mla_status mla_harness_consume(const void* q_out, const void* cache, const int64_t* slot_mapping, int64_t T,
                               int64_t H, int64_t cache_rows, uint32_t flags, float* scores, mla_stream_t stream) {
  using namespace mla::harness;
  if ((flags & ~(MLA_FLAG_Q_FP8 | MLA_FLAG_KV_FP8 | MLA_FLAG_PDL)) != 0) return MLA_ERR_UNSUPPORTED;
  if (T < 0 || H < 1 || cache_rows < 0 || T > (INT64_C(1) << 31) / H) return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  if (!q_out || !slot_mapping || !scores || (!cache && cache_rows > 0)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_out) || (cache && !aligned16(cache)) || (reinterpret_cast<uintptr_t>(scores) & 3u) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return MLA_ERR_ALIGNMENT;
  int32_t sms = 0;
  const mla_status s = mla::current_device(nullptr, &sms);
  if (s != MLA_OK) return s;
  const int64_t rows = T * H;
  int64_t blocks = (rows + 7) / 8;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  const bool qf8 = (flags & MLA_FLAG_Q_FP8) != 0, kvf8 = (flags & MLA_FLAG_KV_FP8) != 0;
  const void* fn = qf8 ? (kvf8 ? reinterpret_cast<const void*>(&consume_kernel<true, true>)
                               : reinterpret_cast<const void*>(&consume_kernel<true, false>))
                       : (kvf8 ? reinterpret_cast<const void*>(&consume_kernel<false, true>)
                               : reinterpret_cast<const void*>(&consume_kernel<false, false>));
  const uint8_t* q = static_cast<const uint8_t*>(q_out);
  const uint8_t* c = static_cast<const uint8_t*>(cache);
  void* args[] = {&q, &c, &slot_mapping, &T, &H, &cache_rows, &scores};
  return launch(fn, dim3(static_cast<unsigned>(blocks)), dim3(256), (flags & MLA_FLAG_PDL) != 0,
                reinterpret_cast<cudaStream_t>(stream), args);
}

}  // extern "C"
