/*
 * mla_epilogue.h -- C ABI of the fused MLA decode epilogue for NVIDIA B200 (sm_100a).
 *
 * The operation (vLLM PR #54896 report on prhub.com.cn, sections 实现拆解
 * "implementation" items 1-3 and 关键源码片段 "key source snippets":
 * fusedKimiK3MLADecodeQConcatKVCacheKernel / writeLatent576 and the
 * launcher fused_kimi_k3_mla_decode_q_concat_kv_cache_insert):
 *
 *   for every token t < T:
 *     for every head h < H:   q_out[t, h, :]            = enc_q (rope(q_nope[t, h, :] || q_pe[t, h, :]))
 *     if slot_mapping[t] ok:  cache.row(slot_mapping[t]) = enc_kv(rope(kv_c[t, :]    || k_pe[t, :]))
 *
 * where every row is 576 = 512 (latent "nope") + 64 (rotary "pe") wide;
 * rope() turns each pair (x[512+i], x[544+i]), i < 32, of the pe part by the
 * angle whose cosine and sine are cos_sin[positions[t]][i] and
 * cos_sin[positions[t]][32+i] (rotate-half RoPE, computed in fp32 as
 * (a c - b s, b c + a s), each product and the sum rounded separately) and
 * leaves the 512 nope values unchanged; enc is a round-to-nearest-even bf16
 * store, or, with the matching FP8 flag, the OCP E4M3FN byte
 * satfinite_rn(y / scale) of the fp32 value y (IEEE fp32 division, no
 * intermediate bf16 rounding).  Without RoPE and FP8 the call is a plain
 * concatenation plus cache scatter, bit for bit.
 *
 * Conventions for every entry point below:
 *   - all data pointers are DEVICE pointers; the caller allocates and owns
 *     every buffer; no entry point allocates, frees or synchronises;
 *   - work is enqueued on `stream` (0 = the legacy default stream) and runs
 *     asynchronously; a return of MLA_OK means "launched", not "finished";
 *   - strides are in ELEMENTS; the innermost stride of every row is 1;
 *   - host-side argument errors return a status and launch nothing.  Index
 *     values that live in device memory (slots, positions) are range-checked
 *     by the kernel, which skips what is out of range and reports it through
 *     the optional status word; it never faults or traps on them.
 */
#ifndef MLA_EPILOGUE_H
#define MLA_EPILOGUE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

/* Same type as cudaStream_t, declared here so that this header needs no CUDA include. */
typedef struct CUstream_st* mla_stream_t;

typedef enum mla_status {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null pointer, negative or too-large size, bad stride, conflicting flags */
  MLA_ERR_ALIGNMENT = 2,   /* a pointer or stride breaks the alignment rules below */
  MLA_ERR_UNSUPPORTED = 3, /* an unknown flag bit */
  MLA_ERR_CUDA = 4         /* the CUDA runtime refused the launch; see mla_last_cuda_error() */
} mla_status;

/* flags */
#define MLA_FLAG_ROPE        1u  /* rotate the 64 pe dims (needs positions, cos_sin) */
#define MLA_FLAG_Q_FP8       2u  /* q_out is e4m3 bytes, scaled by *q_scale (needs q_scale) */
#define MLA_FLAG_KV_FP8      4u  /* cache is e4m3 bytes, scaled by *kv_scale (needs kv_scale) */
#define MLA_FLAG_PDL         8u  /* launch as a programmatic dependent of the previous kernel on `stream` */
#define MLA_FLAG_FORCE_SPLIT 16u /* use MLA_MODE_SPLIT whatever T is (tests, tuning) */
#define MLA_FLAG_FORCE_ROWS  32u /* use MLA_MODE_ROWS whatever T is (tests, tuning); not with FORCE_SPLIT */

/* bits the kernel ORs into *status */
#define MLA_STATUS_SLOT_RANGE 1  /* some slot_mapping[t] >= num_blocks*block_size: that cache row was not written */
#define MLA_STATUS_POS_RANGE  2  /* some positions[t] outside [0, rope_rows): that token's rows were not rotated */
#define MLA_STATUS_TIMEOUT    4  /* a bounded wait inside a kernel (on a copy, a barrier or the tensor cores)
                                    ran out: the outputs are incomplete.  No such wait is expected ever to run
                                    out; the kernel returns instead of hanging */

/* Kernel choice (mla_plan.mode). */
#define MLA_MODE_SPLIT 1 /* small T: three warps per 576-wide row (two move 16-byte nope chunks, one rotates the
                            32 RoPE pairs, one per lane); rows_per_block rows per block, ceil(rows / SMs) up to 4
                            unless tuned, so a single token's rows run one per SM */
#define MLA_MODE_ROWS  2 /* large T: grid-stride over rows, grid sized to the resident blocks; one warp per row
                            (bf16 outputs) or half a warp per row (an e4m3 output) */

/*
 * mla_epilogue_launch -- the whole epilogue in one kernel launch.
 *
 *   q_nope   bf16 [T, H, 512] at element strides (q_nope_stride_t, q_nope_stride_h, 1)
 *   q_pe     bf16 [T, H, 64]  at (q_pe_stride_t, q_pe_stride_h, 1)
 *   kv_c     bf16 [T, 512]    at (kv_c_stride_t, 1)
 *   k_pe     bf16 [T, 64]     at (k_pe_stride_t, 1)
 *   slot_mapping  int64 [T]: cache row (block * block_size + offset) for token t.
 *            A negative slot skips that token's cache row silently; a slot
 *            >= num_blocks*block_size skips it and sets MLA_STATUS_SLOT_RANGE.
 *            Two tokens with the same slot: which row lands is unspecified.
 *   positions int32 [T] and cos_sin fp32 [rope_rows, 64] (row p = cos_0..31 |
 *            sin_0..31 at position p): read only with MLA_FLAG_ROPE (may be
 *            NULL otherwise).  One position per token, shared by its H query
 *            rows and its cache row.  A position outside [0, rope_rows) leaves
 *            that token's rows unrotated and sets MLA_STATUS_POS_RANGE.
 *   q_scale, kv_scale  one fp32 each in device memory (read by the kernel, so
 *            an upstream kernel may write them); read only with the matching
 *            FP8 flag (may be NULL otherwise).  For any scale the e4m3
 *            byte is that of the IEEE fp32 quotient x / scale (the kernel
 *            computes that quotient bit for bit whenever |x| >= 2^-100 and
 *            |x / scale| < 448; outside, both round to the same signed
 *            zero or to +-448).
 *   T >= 0 tokens (T == 0: nothing is launched, MLA_OK); H >= 1 heads;
 *   block_size >= 1, num_blocks >= 0: cache geometry.
 *   q_out    [T, H, 576] contiguous; bf16, or e4m3 bytes with MLA_FLAG_Q_FP8.
 *   cache    [num_blocks, block_size, 576] contiguous; bf16, or e4m3 bytes with
 *            MLA_FLAG_KV_FP8.  Only the T addressed rows are written; every
 *            other byte is left as it was.
 *   status   optional int32 in device memory (NULL = no reporting); the kernel
 *            ORs MLA_STATUS_* bits into it and never clears it.
 *
 * Alignment (the 16-byte row rule of the vLLM PR #54565 report, section 实现拆解
 * item 1): q_nope, kv_c, q_out and cache start on 16-byte boundaries and the
 * strides of q_nope and kv_c are multiples of 8 elements (a stride is not
 * checked when its dimension has size 1); q_pe and k_pe need only bf16
 * (2-byte) alignment; slot_mapping 8 bytes; positions, cos_sin, scales and
 * status 4 bytes.  Strides must be >= 0.  Otherwise MLA_ERR_ALIGNMENT or
 * MLA_ERR_INVALID_ARG and nothing is launched.  Sizes: H <= 65536 and
 * T * (H + 1) < 2^31.  With q_pe and k_pe rows 4-byte aligned (even strides)
 * and cos_sin 8-byte aligned, MLA_MODE_ROWS with an e4m3 output reads and
 * writes the pe values as vectors; the results are the same either way.
 *
 * Programmatic dependent launch (MLA_FLAG_PDL, as the enable_pdl argument of
 * the vLLM PR #54565 report's GEMM entry): the kernel may start before the
 * previous kernel on `stream` has finished.  Query rows wait for it
 * (griddepcontrol.wait) only right before reading q_nope / q_pe; cache rows,
 * slot_mapping, positions, cos_sin and the scales are read without waiting
 * (PR #54896 report, 实现拆解 item 2).  CONTRACT: with this flag the previous
 * kernel on `stream` may write q_nope and q_pe only, and must not read q_out
 * or the cache rows this call writes (cache rows are written while that
 * kernel may still be running).  The kernel signals its own
 * dependents (griddepcontrol.launch_dependents) only after all of its stores
 * (PR #54896 report, 评论区精华: the early trigger was a race and was moved
 * back to the end).
 */
MLA_API mla_status mla_epilogue_launch(
    const void* q_nope, int64_t q_nope_stride_t, int64_t q_nope_stride_h,
    const void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
    const void* kv_c, int64_t kv_c_stride_t,
    const void* k_pe, int64_t k_pe_stride_t,
    const int64_t* slot_mapping,
    const int32_t* positions,
    const float* cos_sin, int64_t rope_rows,
    const float* q_scale, const float* kv_scale,
    int64_t T, int64_t H, int64_t block_size, int64_t num_blocks,
    uint32_t flags,
    void* q_out,
    void* cache,
    int32_t* status,
    mla_stream_t stream);

/*
 * mla_plan -- the launch mla_epilogue_launch would make for (T, H, flags) on
 * the current device, without launching anything.  Host only; needs the
 * device's SM count, which it reads once per device (sm_count <= 0 lets the
 * caller pass it instead: `sm_count` > 0 is used as given and no CUDA call is
 * made).  Returns MLA_ERR_INVALID_ARG for T < 1, H < 1 or both FORCE flags.
 */
typedef struct mla_plan {
  int32_t mode;              /* MLA_MODE_SPLIT or MLA_MODE_ROWS */
  int32_t threads_per_block;
  int64_t blocks;
  int32_t rows_per_block;    /* SPLIT: rows one block covers (96 threads each); ROWS: rows one warp converts at
                                a time (1, or 2 with an e4m3 output) */
  int32_t sm_count;
} mla_plan;

MLA_API mla_status mla_epilogue_plan(int64_t T, int64_t H, uint32_t flags, int32_t sm_count, mla_plan* out);

/*
 * Tuning knobs of the plan (process-wide; not synchronised, set them before
 * launching from several threads).  The pages choose the small-batch split
 * for up to 64 tokens and note that the threshold may not suit other batch
 * sizes or hardware (PR #54896 report, 风险与影响 "risks" item 2).  On B200
 * the split kernel stays faster than the rows kernel up to about 4.6 K rows
 * (T * (H + 1)) whatever H is (measured for H = 8, 16, 32, 128), so the
 * default threshold counts rows, not tokens.
 *   split_max_rows       T * (H + 1) at or below which MLA_MODE_SPLIT is used (default 4608)
 *   split_rows_per_block rows per block in MLA_MODE_SPLIT (block = 96 * this), at most
 *                        10; 0 (default) takes ceil(rows / SMs), at most 4; a negative
 *                        value restores the default
 *   rows_warps_per_block warps per block in MLA_MODE_ROWS, at most 8 (default 8)
 *   rows_blocks_per_sm   blocks per SM the MLA_MODE_ROWS grid is sized for, at most
 *                        the number the kernel's register cap keeps resident (4 with
 *                        an e4m3 output, 5 without; default: that number)
 * Larger values are clamped to those limits; 0 keeps the current setting.
 */
typedef struct mla_tuning {
  int64_t split_max_rows;
  int32_t split_rows_per_block;
  int32_t rows_warps_per_block;
  int32_t rows_blocks_per_sm;
} mla_tuning;

MLA_API void mla_epilogue_set_tuning(const mla_tuning* t);
MLA_API void mla_epilogue_get_tuning(mla_tuning* out);

/* Text for a status code (static storage). */
MLA_API const char* mla_status_string(mla_status s);

/* The cudaError_t of the last launch that returned MLA_ERR_CUDA on this host thread (0 if none). */
MLA_API int32_t mla_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_EPILOGUE_H */
