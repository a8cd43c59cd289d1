/*
 * mla_absorb.h -- the query side of the fused MLA decode epilogue with its
 * producer folded in, on the tcgen05 tensor cores of B200 (sm_100a).
 *
 * In MLA decode with weight absorption the 512 latent ("nope") values of a
 * query row are the product of the 128-wide nope query of that head with
 * the head's absorbed key weight; the epilogue then concatenates them with
 * the 64 rotary values (vLLM PR #54896 report, 实现拆解 item 2: the epilogue
 * sits behind the upstream GEMM).  This entry point computes that product
 * and writes the finished latent query rows in one kernel, so the 512-wide
 * intermediate never goes through memory:
 *
 *   q_out[t, h, j]       = enc( sum_k q_nope_c[t, h, k] * w_uk[h, j, k] ),  j < 512, k < 128
 *   q_out[t, h, 512 + i] = enc( rope(q_pe[t, h, :])[i] ),                   i < 64
 *
 * with enc and rope exactly as in mla_epilogue.h (bf16 round to nearest
 * even, or e4m3 of x / *q_scale; rotate-half over (i, i+32) with
 * cos_sin[positions[t]]).  The products accumulate in fp32 on the tensor
 * cores (order unspecified), so the 512 nope values match an exact dot
 * product within fp32 accumulation error before encoding; the 64 pe values
 * are bit-identical to mla_epilogue_launch's.  The cache row is not written
 * here (mla_epilogue_launch does it).
 *
 * Same conventions as mla_epilogue.h: device pointers owned by the caller,
 * element strides, asynchronous on `stream`, nothing allocated, host errors
 * returned as mla_status before anything is launched.
 */
#ifndef MLA_ABSORB_H
#define MLA_ABSORB_H

#include <stdint.h>

#include "mla_epilogue.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * mla_absorb_launch
 *   q_nope_c  bf16 [T, H, 128] at element strides (stride_t, stride_h, 1): the
 *             nope query before absorption.  16-byte aligned; strides
 *             multiples of 8 elements (unchecked for a size-1 dimension).
 *   w_uk      bf16 [H, 512, 128] contiguous, 16-byte aligned: per head, the 512
 *             latent rows of 128 (row j holds the weights of latent value j).
 *   q_pe      bf16 [T, H, 64] at (q_pe_stride_t, q_pe_stride_h, 1), 2-byte aligned.
 *   positions, cos_sin, rope_rows, q_scale: as in mla_epilogue_launch
 *             (flags MLA_FLAG_ROPE, MLA_FLAG_Q_FP8).
 *   T >= 0, 1 <= H <= 65535, T * H <= 2^31 - 1 - 128.
 *   q_out     [T, H, 576] contiguous, bf16 or e4m3 bytes, 16-byte aligned.
 *   status    optional device int32: MLA_STATUS_POS_RANGE, MLA_STATUS_TIMEOUT.
 *   flags     MLA_FLAG_ROPE, MLA_FLAG_Q_FP8, MLA_FLAG_PDL (the q inputs come
 *             from the previous kernel on `stream`: the weights, positions,
 *             table and scale are read before waiting for it; the kernel
 *             triggers its own dependents after its last store).
 * Errors: MLA_ERR_INVALID_ARG, MLA_ERR_ALIGNMENT, MLA_ERR_UNSUPPORTED (flag
 * bits), MLA_ERR_CUDA (launch refused, or the driver's tensor-map encoder is
 * unavailable).
 */
MLA_API mla_status mla_absorb_launch(
    const void* q_nope_c, int64_t q_nope_c_stride_t, int64_t q_nope_c_stride_h,
    const void* w_uk,
    const void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
    const int32_t* positions, const float* cos_sin, int64_t rope_rows,
    const float* q_scale,
    int64_t T, int64_t H, uint32_t flags,
    void* q_out, int32_t* status, mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_ABSORB_H */
