/*
 * mla_harness.h -- measurement and self-check kernels that sit beside the
 * fused MLA decode epilogue (same library as mla_epilogue.h, same
 * conventions: device pointers owned by the caller, asynchronous on
 * `stream`, nothing allocated, host argument errors returned as mla_status).
 *
 * None of these is part of the epilogue itself.  They put it in the setting
 * the vLLM PR #54896 report describes: an upstream producer kernel, linked
 * by programmatic dependent launch (实现拆解 item 2), and a downstream
 * consumer.  They also time a bare launch, and check the e4m3 quotient on
 * the device.
 */
#ifndef MLA_HARNESS_H
#define MLA_HARNESS_H

#include <stdint.h>

#include "mla_epilogue.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Synthetic upstream producer: writes q_nope [T,H,512] and q_pe [T,H,64]
 * (bf16, strides as in mla_epilogue_launch) by copying src_nope [T,H,512] and
 * src_pe [T,H,64] (contiguous bf16), standing in for the projection GEMM
 * that produces the latent query (PR #54896 report, 实现拆解 item 2: the
 * epilogue sits between an upstream GEMM and the attention kernel).  Each of
 * its blocks signals griddepcontrol.launch_dependents when it starts, so a
 * dependent launched with MLA_FLAG_PDL can be scheduled while it runs; the
 * dependent's griddepcontrol.wait still waits for all of its stores.
 * flags: MLA_FLAG_PDL (this launch itself is a programmatic dependent) only.
 * Alignment: every pointer 16 bytes, strides multiples of 8 elements.
 */
MLA_API mla_status mla_harness_produce(const void* src_nope, const void* src_pe,
                               void* q_nope, int64_t q_nope_stride_t, int64_t q_nope_stride_h,
                               void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
                               int64_t T, int64_t H, uint32_t flags, mla_stream_t stream);

/*
 * The same producer with the duration of a real one: before it writes q it
 * reads `weight_bytes` of `weights` through all of its blocks, as the
 * projection GEMM streams its weight matrix before its epilogue writes the
 * query (PR #54896 report, 实现拆解 item 2: the epilogue's loads that do not
 * depend on the GEMM overlap the GEMM's tail).  Every block XORs the 32-bit
 * words it read into *sink (device, 4-byte aligned), so after one call *sink
 * is its old value XOR every word of the weights.  The grid covers all SMs
 * (4 blocks of 256 threads each) however small T is.  weights: 16-byte
 * aligned, weight_bytes a multiple of 16 (0 reads nothing).  Otherwise as
 * mla_harness_produce.
 */
MLA_API mla_status mla_harness_produce_after_weights(const void* src_nope, const void* src_pe,
                               void* q_nope, int64_t q_nope_stride_t, int64_t q_nope_stride_h,
                               void* q_pe, int64_t q_pe_stride_t, int64_t q_pe_stride_h,
                               const void* weights, int64_t weight_bytes, uint32_t* sink,
                               int64_t T, int64_t H, uint32_t flags, mla_stream_t stream);

/*
 * An empty kernel launched with `blocks` x `threads` and, with MLA_FLAG_PDL,
 * the programmatic-serialization attribute: the bare-launch floor that the
 * epilogue's latency at decode sizes is compared with.  With
 * MLA_HARNESS_EMPTY_WAIT every thread executes griddepcontrol.wait and then
 * exits: the cheapest kernel that honours a programmatic dependency, i.e. the
 * floor of a dependent launch behind an upstream kernel.
 */
#define MLA_HARNESS_EMPTY_WAIT 256u
MLA_API mla_status mla_harness_empty(int64_t blocks, int32_t threads, uint32_t flags, mla_stream_t stream);

/*
 * Device check of the e4m3 quotient: for every fp32 bit pattern p in
 * [first, first + count) compares the epilogue's quotient x / scale with the
 * CUDA IEEE division __fdiv_rn (NaN equal to NaN), and the e4m3 bytes the
 * epilogue stores with those of the IEEE quotient, both for x as an fp32
 * (the rotated pe values) and for the two halves of p as bf16 (the other
 * values).  result (device, 3 x uint64, overwritten): [0] inputs with
 * |x| >= 2^-100 and |x / scale| < 448 whose quotients differ (outside that
 * range the epilogue's quotient may differ in its last bits while its e4m3
 * byte, a signed zero below and +-448 above, may not), [1] patterns whose
 * e4m3 bytes differ on either path, [2] smallest pattern counted in [0] or
 * [1] (UINT64_MAX if none).  first + count <= 2^32.
 */
MLA_API mla_status mla_harness_div_check(float scale, uint64_t first, uint64_t count,
                                 unsigned long long* result, mla_stream_t stream);

/*
 * Device check of the e4m3 bytes of bf16 inputs over many scales: for every
 * scale bit pattern in [first, first + count) and every one of the 65536
 * bf16 values x, compares the e4m3 byte the epilogue stores for x / scale
 * with the byte of CUDA's IEEE quotient __fdiv_rn.  (The epilogue reaches
 * bf16 quotients in one corrected step; they may differ from the IEEE
 * quotient in the last bit but not in the e4m3 byte.)  result (device,
 * 2 x uint64, 8-byte aligned, overwritten): [0] differing (scale, x) pairs,
 * [1] smallest scale pattern with one (UINT64_MAX if none).
 * first + count <= 2^32.  Work: count x 65536 quotients per call.
 */
MLA_API mla_status mla_harness_bf16_scale_check(uint32_t first, uint32_t count, unsigned long long* result,
                                                mla_stream_t stream);

/*
 * Synthetic downstream consumer standing in for the attention kernel that
 * reads the epilogue's outputs (PR #54896 report, 实现拆解 item 2: the
 * epilogue's trigger lets the attention kernel overlap with it).  For every
 * token t and head h it writes
 *     scores[t * H + h] = sum_i dec(q_out[t, h, i]) * dec(cache.row(slot_mapping[t])[i])
 * in fp32 (dec: bf16, or e4m3 with MLA_FLAG_Q_FP8 / MLA_FLAG_KV_FP8; the
 * scales are not applied), or NaN when the slot is outside
 * [0, cache_rows).  It reads slot_mapping before its griddepcontrol.wait
 * and q_out and the cache only after it, so, launched with MLA_FLAG_PDL
 * right behind the epilogue, it sees every store the epilogue made.
 * q_out and cache: 16-byte aligned; scores: fp32 [T * H], 4-byte aligned.
 */
MLA_API mla_status mla_harness_consume(const void* q_out, const void* cache, const int64_t* slot_mapping,
                                       int64_t T, int64_t H, int64_t cache_rows, uint32_t flags, float* scores,
                                       mla_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MLA_HARNESS_H */
