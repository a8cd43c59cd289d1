// mla_oracle.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, single-threaded CPU oracle of the fused MLA decode epilogue
// (mla_oracle_run_threads only runs that same function on token slices in
// parallel, for the benchmark's all-cores baseline):
// per token it builds H latent query rows and one latent KV-cache row, each
// 576 wide, exactly as the operation is defined, with no blocking, fusion or
// reordering.  Only the tests, the smoke check and the benchmark's CPU
// baseline may load this library; the product path never does.  It shares no
// code (kernels, headers, helpers, tables) with the CUDA library.
//
// Sources (all from the prhub.com.cn reports on vLLM pull requests):
//   * vLLM PR #54896 report, section "实现拆解" (implementation) items 1-3 and
//     the "关键源码片段" (key source) listing of fusedKimiK3MLADecodeQConcat-
//     KVCacheKernel / writeLatent576: one 576-wide latent row per (token, head)
//     plus one cache row per token, optional RoPE on the 64 pe dims and
//     optional FP8 output for Q and for KV (template flags Q_FP8, KV_FP8,
//     APPLY_ROPE).
//   * same report, key-source listing of test_decode_epilogue_row_split_boundary:
//     q == cat(ql_nope, q_pe) and cache rows at slot_mapping == cat(kv_c, k_pe)
//     when neither RoPE nor FP8 is on.
// Readings where the pages are silent:
//   * RoPE is rotate-half over the pairs (i, i+32) of the 64 pe dims, with a
//     fp32 table row [cos_0..cos_31 | sin_0..sin_31] per position; one position
//     per token, shared by all of its rows.  Computed in fp32, no contraction.
//   * FP8 is OCP E4M3FN, per-tensor scale, byte = satfinite_rn(y / scale) with
//     IEEE fp32 division, quantised straight from the fp32 value.
//   * rows that are not rotated and not quantised are bf16 copies.
//   * slot < 0: the cache row is not written.  slot >= num_blocks*block_size:
//     not written, status bit 1.  RoPE position outside [0, rope_rows): the
//     token's rows are written unrotated, status bit 2.
//
// Build: g++ -O2 -ffp-contract=off -fno-fast-math (see build.py).  The
// arithmetic below relies on no fused multiply-add and on SSE (not x87)
// single precision, which is the x86-64 default.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

constexpr int kNope = 512;
constexpr int kPe = 64;
constexpr int kHalfPe = 32;
constexpr int kRow = kNope + kPe;  // 576

constexpr uint32_t kFlagRope = 1u;
constexpr uint32_t kFlagQFp8 = 2u;
constexpr uint32_t kFlagKvFp8 = 4u;

constexpr int32_t kStatusSlotRange = 1;
constexpr int32_t kStatusPosRange = 2;

float f32_from_bits(uint32_t u) {
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

uint32_t bits_from_f32(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return u;
}

// bf16 -> fp32: a bf16 value is the top half of an fp32 word, so this is exact.
float bf16_to_f32(uint16_t h) { return f32_from_bits(static_cast<uint32_t>(h) << 16); }

// fp32 -> bf16, round to nearest, ties to even.  bf16 keeps the fp32 sign and
// 8-bit exponent and the top 7 fraction bits; the dropped 16 bits decide the
// rounding.  NaN keeps its top bits (so a bf16 NaN that went through fp32
// unchanged comes back bit for bit) and is forced quiet if they would read as
// infinity.
uint16_t f32_to_bf16_rne(float f) {
  const uint32_t u = bits_from_f32(f);
  if ((u & 0x7fffffffu) > 0x7f800000u) {
    uint16_t top = static_cast<uint16_t>(u >> 16);
    if ((top & 0x7fu) == 0) top |= 0x40u;
    return top;
  }
  const uint32_t upper = u >> 16;
  const uint32_t lower = u & 0xffffu;
  uint32_t out = upper;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) out += 1;  // may carry into the exponent: correct, up to inf
  return static_cast<uint16_t>(out);
}

// Round a non-negative double that holds an exactly known value to the
// nearest integer, ties to even.
double round_half_even(double x) {
  const double fl = std::floor(x);
  const double frac = x - fl;
  if (frac > 0.5) return fl + 1.0;
  if (frac < 0.5) return fl;
  return (std::fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

// fp32 -> OCP FP8 E4M3FN, round to nearest even, saturating to the largest
// finite value.  Format: 1 sign, 4 exponent (bias 7), 3 fraction bits; no
// infinity; S.1111.111 is NaN, so the largest finite is S.1111.110 = 448.
// Normal values 2^(E-7) * (1 + k/8), E in 1..15; subnormals k * 2^-9.
// Saturation happens after rounding: everything at or above 448 (including
// infinity) maps to 448 with the input's sign; zero keeps its sign.
uint8_t f32_to_e4m3_satfinite(float f) {
  const uint32_t u = bits_from_f32(f);
  const uint8_t sign = static_cast<uint8_t>((u >> 24) & 0x80u);
  if (std::isnan(f)) return static_cast<uint8_t>(sign | 0x7fu);
  const double a = std::fabs(static_cast<double>(f));  // exact
  if (a >= 448.0) return static_cast<uint8_t>(sign | 0x7eu);
  if (a < 0.015625) {  // below 2^-6: subnormal grid of step 2^-9
    const double k = round_half_even(a * 512.0);  // exact scaling by 2^9
    // k == 8 is 2^-6, the smallest normal, whose encoding 0x08 is also k.
    return static_cast<uint8_t>(sign | static_cast<uint8_t>(k));
  }
  int e2 = 0;
  const double m = std::frexp(a, &e2);  // a = m * 2^e2, m in [0.5, 1)
  int e = e2 - 1;                       // a = (2m) * 2^e, 2m in [1, 2)
  double k = round_half_even((2.0 * m - 1.0) * 8.0);  // exact: 2m has <= 24 significant bits
  if (k >= 8.0) {
    k = 0.0;
    e += 1;
  }
  if (e > 8 || (e == 8 && k > 6.0)) return static_cast<uint8_t>(sign | 0x7eu);
  return static_cast<uint8_t>(sign | static_cast<uint8_t>((e + 7) << 3) | static_cast<uint8_t>(k));
}

// One latent row from 512 fp32 nope values and 64 bf16 pe values: the pe
// part optionally rotated, then all 576 encoded to bf16 or to e4m3.
void encode_latent_row(const float* nope, const uint16_t* pe, const float* rope_row,
                       bool fp8, float scale, uint8_t* dst) {
  float x[kRow];
  for (int i = 0; i < kNope; ++i) x[i] = nope[i];
  for (int i = 0; i < kPe; ++i) x[kNope + i] = bf16_to_f32(pe[i]);

  float y[kRow];
  for (int i = 0; i < kRow; ++i) y[i] = x[i];
  if (rope_row != nullptr) {
    // rotate-half: the pair (i, i+32) of the pe dims turns by angle theta_i.
    for (int i = 0; i < kHalfPe; ++i) {
      const float c = rope_row[i];
      const float s = rope_row[kHalfPe + i];
      const float a = x[kNope + i];
      const float b = x[kNope + kHalfPe + i];
      const float ac = a * c;
      const float bs = b * s;
      const float bc = b * c;
      const float as = a * s;
      y[kNope + i] = ac - bs;
      y[kNope + kHalfPe + i] = bc + as;
    }
  }

  if (fp8) {
    for (int i = 0; i < kRow; ++i) {
      const float q = y[i] / scale;  // IEEE single-precision division
      dst[i] = f32_to_e4m3_satfinite(q);
    }
  } else {
    for (int i = 0; i < kRow; ++i) {
      const uint16_t h = f32_to_bf16_rne(y[i]);
      std::memcpy(dst + 2 * i, &h, sizeof h);
    }
  }
}

// One latent row from bf16 sources (the epilogue's rows).
void build_latent_row(const uint16_t* nope, const uint16_t* pe, const float* rope_row,
                      bool fp8, float scale, uint8_t* dst) {
  float x[kNope];
  for (int i = 0; i < kNope; ++i) x[i] = bf16_to_f32(nope[i]);
  encode_latent_row(x, pe, rope_row, fp8, scale, dst);
}

}  // namespace

extern "C" {

// Element conversions, exported so the tests can pin them one by one.
float mla_oracle_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }
uint16_t mla_oracle_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
uint8_t mla_oracle_f32_to_e4m3(float f) { return f32_to_e4m3_satfinite(f); }

// The whole epilogue over host buffers.  Argument meanings mirror the
// product entry point (element strides; inner strides are 1):
//   q_nope [T,H,512] bf16 at strides (qn_st, qn_sh); q_pe [T,H,64] at (qp_st, qp_sh)
//   kv_c [T,512] at kv_st; k_pe [T,64] at kp_st
//   slot_mapping [T] int64; positions [T] int32 and cos_sin [rope_rows,64] fp32 (RoPE only)
//   q_scale / kv_scale: one fp32 each (FP8 only)
//   q_out [T,H,576] contiguous, bf16 (2 B) or e4m3 (1 B) per element
//   cache [num_blocks*block_size, 576] contiguous, bf16 or e4m3
//   *status receives the OR of the status bits (may be null).
// Returns 0, or 1 when an argument is unusable (nothing is written then).
int mla_oracle_run(const uint16_t* q_nope, int64_t qn_st, int64_t qn_sh,
                   const uint16_t* q_pe, int64_t qp_st, int64_t qp_sh,
                   const uint16_t* kv_c, int64_t kv_st,
                   const uint16_t* k_pe, int64_t kp_st,
                   const int64_t* slot_mapping, const int32_t* positions,
                   const float* cos_sin, int64_t rope_rows,
                   const float* q_scale, const float* kv_scale,
                   int64_t T, int64_t H, int64_t block_size, int64_t num_blocks,
                   uint32_t flags, void* q_out, void* cache, int32_t* status) {
  if (T < 0 || H < 1 || block_size < 1 || num_blocks < 0) return 1;
  if ((flags & ~(kFlagRope | kFlagQFp8 | kFlagKvFp8)) != 0) return 1;
  if (T == 0) return 0;  // nothing to read or write
  const bool rope = (flags & kFlagRope) != 0;
  const bool q_fp8 = (flags & kFlagQFp8) != 0;
  const bool kv_fp8 = (flags & kFlagKvFp8) != 0;
  if (rope && (positions == nullptr || cos_sin == nullptr || rope_rows < 1)) return 1;
  if (q_fp8 && q_scale == nullptr) return 1;
  if (kv_fp8 && kv_scale == nullptr) return 1;
  const int64_t cache_rows = num_blocks * block_size;

  int32_t st = 0;
  uint8_t* qo = static_cast<uint8_t*>(q_out);
  uint8_t* kc = static_cast<uint8_t*>(cache);
  const int64_t q_row_bytes = q_fp8 ? kRow : 2 * kRow;
  const int64_t kv_row_bytes = kv_fp8 ? kRow : 2 * kRow;

  for (int64_t t = 0; t < T; ++t) {
    const float* rope_row = nullptr;
    if (rope) {
      const int64_t pos = positions[t];
      if (pos >= 0 && pos < rope_rows) {
        rope_row = cos_sin + pos * kPe;
      } else {
        st |= kStatusPosRange;
      }
    }
    for (int64_t r = 0; r < H; ++r) {
      const uint16_t* nope = q_nope + t * qn_st + r * qn_sh;
      const uint16_t* pe = q_pe + t * qp_st + r * qp_sh;
      uint8_t* dst = qo + (t * H + r) * q_row_bytes;
      build_latent_row(nope, pe, rope_row, q_fp8, q_fp8 ? *q_scale : 1.0f, dst);
    }
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= cache_rows) {
      st |= kStatusSlotRange;
      continue;
    }
    build_latent_row(kv_c + t * kv_st, k_pe + t * kp_st, rope_row, kv_fp8,
                     kv_fp8 ? *kv_scale : 1.0f, kc + slot * kv_row_bytes);
  }
  if (status != nullptr) *status |= st;
  return 0;
}

// Latent query rows from the absorption product (the query side of the
// epilogue with its producer folded in).  For every token t and head h:
//   ql[j] = sum_k q_nope_c[t, h, k] * w_uk[h, j, k],  j < 512, k < 128
// accumulated in double precision in k order (every bf16 x bf16 product is
// exact in double; the running sum carries 53 bits) and rounded once to
// fp32; then the row [ql | rope(q_pe[t, h])] is encoded like every other
// query row.
//   q_nope_c [T,H,128] bf16 at (qc_st, qc_sh); w_uk [H,512,128] bf16 contiguous
//   q_pe [T,H,64] at (qp_st, qp_sh); positions / cos_sin / q_scale as in mla_oracle_run
//   q_out [T,H,576] contiguous, bf16 or e4m3 (flag Q_FP8).
// flags: ROPE, Q_FP8 only.  Returns 0, or 1 for an unusable argument.
int mla_oracle_absorb_run(const uint16_t* q_nope_c, int64_t qc_st, int64_t qc_sh, const uint16_t* w_uk,
                          const uint16_t* q_pe, int64_t qp_st, int64_t qp_sh, const int32_t* positions,
                          const float* cos_sin, int64_t rope_rows, const float* q_scale, int64_t T, int64_t H,
                          uint32_t flags, void* q_out, int32_t* status) {
  if (T < 0 || H < 1) return 1;
  if ((flags & ~(kFlagRope | kFlagQFp8)) != 0) return 1;
  if (T == 0) return 0;
  const bool rope = (flags & kFlagRope) != 0;
  const bool q_fp8 = (flags & kFlagQFp8) != 0;
  if (rope && (positions == nullptr || cos_sin == nullptr || rope_rows < 1)) return 1;
  if (q_fp8 && q_scale == nullptr) return 1;
  constexpr int kIn = 128;
  int32_t st = 0;
  uint8_t* qo = static_cast<uint8_t*>(q_out);
  const int64_t row_bytes = q_fp8 ? kRow : 2 * kRow;
  float ql[kNope];
  for (int64_t t = 0; t < T; ++t) {
    const float* rope_row = nullptr;
    if (rope) {
      const int64_t pos = positions[t];
      if (pos >= 0 && pos < rope_rows) {
        rope_row = cos_sin + pos * kPe;
      } else {
        st |= kStatusPosRange;
      }
    }
    for (int64_t h = 0; h < H; ++h) {
      const uint16_t* a = q_nope_c + t * qc_st + h * qc_sh;
      for (int j = 0; j < kNope; ++j) {
        const uint16_t* b = w_uk + (h * kNope + j) * kIn;
        double acc = 0.0;
        for (int k = 0; k < kIn; ++k) {
          acc += static_cast<double>(bf16_to_f32(a[k])) * static_cast<double>(bf16_to_f32(b[k]));
        }
        ql[j] = static_cast<float>(acc);
      }
      encode_latent_row(ql, q_pe + t * qp_st + h * qp_sh, rope_row, q_fp8, q_fp8 ? *q_scale : 1.0f,
                        qo + (t * H + h) * row_bytes);
    }
  }
  if (status != nullptr) *status |= st;
  return 0;
}

// The benchmark's all-cores baseline: mla_oracle_run, unchanged, on
// `threads` contiguous token slices at once (one std::thread each).  Tokens
// are independent and the caller's slots are unique, so the slices write
// disjoint rows; nothing is reordered inside a slice.
int mla_oracle_run_threads(const uint16_t* q_nope, int64_t qn_st, int64_t qn_sh,
                           const uint16_t* q_pe, int64_t qp_st, int64_t qp_sh,
                           const uint16_t* kv_c, int64_t kv_st,
                           const uint16_t* k_pe, int64_t kp_st,
                           const int64_t* slot_mapping, const int32_t* positions,
                           const float* cos_sin, int64_t rope_rows,
                           const float* q_scale, const float* kv_scale,
                           int64_t T, int64_t H, int64_t block_size, int64_t num_blocks,
                           uint32_t flags, void* q_out, void* cache, int32_t* status, int threads) {
  if (threads < 1 || T < 0 || H < 1) return 1;
  if (T == 0) return mla_oracle_run(q_nope, qn_st, qn_sh, q_pe, qp_st, qp_sh, kv_c, kv_st, k_pe, kp_st, slot_mapping,
                                    positions, cos_sin, rope_rows, q_scale, kv_scale, T, H, block_size, num_blocks,
                                    flags, q_out, cache, status);
  const int n = static_cast<int>(threads < T ? threads : T);
  const int64_t q_row_bytes = (flags & kFlagQFp8) ? kRow : 2 * kRow;
  std::vector<int32_t> st(n, 0);
  std::vector<int> rc(n, 0);
  std::vector<std::thread> pool;
  for (int i = 0; i < n; ++i) {
    const int64_t t0 = T * i / n, t1 = T * (i + 1) / n;
    pool.emplace_back([=, &st, &rc]() {
      rc[i] = mla_oracle_run(q_nope + t0 * qn_st, qn_st, qn_sh, q_pe + t0 * qp_st, qp_st, qp_sh, kv_c + t0 * kv_st,
                             kv_st, k_pe + t0 * kp_st, kp_st, slot_mapping + t0,
                             positions != nullptr ? positions + t0 : nullptr, cos_sin, rope_rows, q_scale, kv_scale,
                             t1 - t0, H, block_size, num_blocks, flags,
                             static_cast<uint8_t*>(q_out) + t0 * H * q_row_bytes, cache, &st[i]);
    });
  }
  int result = 0;
  for (int i = 0; i < n; ++i) {
    pool[i].join();
    if (rc[i] != 0) result = rc[i];
    if (status != nullptr) *status |= st[i];
  }
  return result;
}

}  // extern "C"
