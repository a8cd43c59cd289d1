"""GPU parity: the CUDA path through the C ABI against the CPU oracle, element
by element, on the same seeded inputs.

The kernels compute every rotated value with explicitly rounded fp32
operations and every e4m3 quotient exactly, so the bar here is bit-exact for
all outputs (stricter than the 1 bf16 ulp / 1 e4m3 step the operation
allows for RoPE'd values).  Untouched cache rows are compared too, since
the whole cache is compared.
"""

import pytest
import torch

from mla_decode_attention_10_b200 import epilogue as E
from mla_decode_attention_10_b200 import workloads as W
from parity_util import assert_same, check_workload, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

FORCE = [0, E.MLA_FLAG_FORCE_SPLIT, E.MLA_FLAG_FORCE_ROWS]


# ---- the named workloads at their full sizes, in the launch configuration the bench times

@pytest.mark.parametrize("name", [n for n in W.names() if n != "batch_t8192_h16_pdl_fp8"])
def test_named_workload_matches_oracle(name):
    w = W.all_named()[name]()
    check_workload(w)


def test_large_batch_behind_producer_with_pdl_matches_oracle():
    w = W.batch_t8192_h16_pdl_fp8()
    check_workload(w, producer=True)


# ---- every kernel on the same inputs: bitwise identical (row split, single token, large batch)

@pytest.mark.parametrize("T", [1, 7, 64, 65, 300])
@pytest.mark.parametrize("flags", [0, W.FLAG_ROPE, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8,
                                   W.FLAG_Q_FP8, W.FLAG_KV_FP8 | W.FLAG_ROPE])
def test_split_and_rows_kernels_agree_with_oracle(T, flags):
    w = W.make("modes", T, 16, flags, seed=T * 31 + flags, num_blocks=16, std=2.0,
               rope_rows=4096, scale=0.05, cache_fill="random")
    qo, co, so = run_oracle(w)
    for f in FORCE[1:]:
        qg, cg, sg = run_gpu(w, extra_flags=f)
        assert sg == so
        assert_same(qg, qo, f"q_out force={f}")
        assert_same(cg, co, f"cache force={f}")


# ---- every flag combination, odd head counts, strided views, ragged tails

@pytest.mark.parametrize("flags", list(range(8)))
@pytest.mark.parametrize("T,H", [(3, 1), (5, 5), (33, 7), (129, 3)])
def test_flag_combinations_and_shapes(flags, T, H):
    w = W.make("combo", T, H, flags, seed=1000 + flags * 17 + T * H, num_blocks=8, block_size=32,
               std=2.0, rope_rows=512, scale=0.37, cache_fill="random",
               q_nope_row=520, q_pe_row=65, kv_c_row=1024, kv_c_offset=504, k_pe_row=67)
    for f in FORCE:
        check_workload(w, extra_flags=f)


# ---- the single-token path (PR #53526 in the PR #54896 report's 关联脉络)

@pytest.mark.parametrize("flags", list(range(8)))
@pytest.mark.parametrize("H", [1, 16, 27, 28, 128])
def test_single_token_behind_producer(flags, H):
    """T = 1 through the plan's own choice (one row per block, spread over
    the SMs), launched with PDL behind the synthetic producer, every flag
    combination."""
    p = E.mla_epilogue_plan(1, H, flags)
    assert p.mode == E.MLA_MODE_SPLIT and p.rows_per_block == 1
    w = W.make("token", 1, H, flags, seed=600 + H * 8 + flags, num_blocks=2, std=2.0, rope_rows=1024,
               scale=0.05, cache_fill="random")
    check_workload(w, producer=True)
    check_workload(w)


# ---- inputs off the 16-byte grid take the scalar pe / table paths

def _shift_view(t: torch.Tensor, elems: int) -> torch.Tensor:
    """The same values in a buffer whose first element sits `elems` elements
    past a 16-byte boundary (contiguous rows, same strides)."""
    flat = torch.empty(t.numel() + elems, dtype=t.dtype)
    out = flat[elems:].view(t.shape)
    out.copy_(t)
    return out


@pytest.mark.parametrize("force", FORCE)
@pytest.mark.parametrize("T", [1, 9, 300])
@pytest.mark.parametrize("pe_shift,k_shift,table_shift", [(1, 3, 1), (2, 2, 1), (2, 6, 2)])
def test_unaligned_pe_rows_and_table(force, T, pe_shift, k_shift, table_shift):
    """q_pe / k_pe rows and the cos/sin table off the 16-byte grid: 2-byte
    aligned pe (one element pairs at a time), 4-byte aligned pe with a 4-byte
    aligned table (still one pair at a time), and 4-byte pe with an 8-byte
    aligned table (the rows kernel takes two pairs per lane)."""
    w = W.make("unaligned", T, 16, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=70 + T, num_blocks=8, std=2.0, rope_rows=512,
               scale=0.05, cache_fill="random")
    w.q_pe = _shift_view(w.q_pe.contiguous(), pe_shift)
    w.k_pe = _shift_view(w.k_pe.contiguous(), k_shift)
    w.cos_sin = _shift_view(w.cos_sin, table_shift)
    assert w.q_pe.data_ptr() % 16 and w.k_pe.data_ptr() % 16 and w.cos_sin.data_ptr() % 16
    check_workload(w, extra_flags=force)


# ---- the large-batch kernel's block shape: any number of consumer warps

@pytest.mark.parametrize("warps", [1, 3, 8])
def test_rows_kernel_warp_counts(warps):
    """Blocks of 1 .. 8 warps; every warp walks many rows."""
    old = E.mla_epilogue_get_tuning()
    try:
        E.mla_epilogue_set_tuning(rows_warps_per_block=warps)
        assert E.mla_epilogue_plan(777, 12, E.MLA_FLAG_FORCE_ROWS).threads_per_block == 32 * warps
        w = W.make("warps", 777, 12, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=90 + warps, num_blocks=64,
                   std=2.0, rope_rows=2048, scale=0.05, cache_fill="random")
        check_workload(w, extra_flags=E.MLA_FLAG_FORCE_ROWS)
        check_workload(w, extra_flags=E.MLA_FLAG_FORCE_ROWS, producer=True)
    finally:
        E.mla_epilogue_set_tuning(old.split_max_rows, old.split_rows_per_block or -1, old.rows_warps_per_block,
                                  old.rows_blocks_per_sm)


@pytest.mark.parametrize("rpb", [1, 3, 10])
def test_split_kernel_rows_per_block(rpb):
    """Blocks of 1 .. 10 rows, the last one ragged."""
    old = E.mla_epilogue_get_tuning()
    try:
        E.mla_epilogue_set_tuning(split_rows_per_block=rpb)
        w = W.make("rpb", 37, 7, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=rpb, num_blocks=8, std=2.0,
                   rope_rows=512, scale=0.05, cache_fill="random")
        assert E.mla_epilogue_plan(37, 7, E.MLA_FLAG_FORCE_SPLIT).rows_per_block == rpb
        check_workload(w, extra_flags=E.MLA_FLAG_FORCE_SPLIT)
        check_workload(w, extra_flags=E.MLA_FLAG_FORCE_SPLIT, producer=True)
    finally:
        E.mla_epilogue_set_tuning(old.split_max_rows, old.split_rows_per_block or -1, old.rows_warps_per_block,
                                  old.rows_blocks_per_sm)


def test_prefill_strided_views_are_really_strided():
    w = W.prefill_t1024_h128_strided()
    assert w.q_nope.stride() == (128 * 640, 640, 1)
    assert w.kv_c.stride() == (1536, 1) and w.kv_c.storage_offset() == 512


# ---- exhaustive element checks

def _all_bf16_patterns():
    return torch.arange(65536, dtype=torch.int32).to(torch.int16)


@pytest.mark.parametrize("scale", [0.05, 1.0, 0.37, 3.0, 7.0, 0.9])
@pytest.mark.parametrize("force", FORCE[1:])
def test_every_bf16_pattern_quantises_like_the_oracle(scale, force):
    """All 65536 bf16 patterns in q_nope and kv_c, Q and KV e4m3: the bytes
    match the oracle's; NaN inputs give an e4m3 NaN (0x7f / 0xff) on both."""
    w = W.make("e4m3", 8, 16, W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=3, num_blocks=1, block_size=16, scale=scale)
    u = _all_bf16_patterns()
    w.q_nope.view(torch.int16).copy_(u.view(8, 16, 512))
    w.kv_c.view(torch.int16).copy_(u[-8 * 512:].view(8, 512))
    qg, cg, _ = run_gpu(w, extra_flags=force)
    qo, co, _ = run_oracle(w)
    nan_in = torch.isnan(torch.cat((w.q_nope, w.q_pe), -1).float())
    assert torch.equal(qg[~nan_in], qo[~nan_in])
    assert torch.all((qg[nan_in] & 0x7F) == 0x7F) and torch.all((qo[nan_in] & 0x7F) == 0x7F)
    kvnan = torch.isnan(torch.cat((w.kv_c, w.k_pe), -1).float())
    rows_g = cg.view(-1, 576)[w.slot_mapping]
    rows_o = co.view(-1, 576)[w.slot_mapping]
    assert torch.equal(rows_g[~kvnan], rows_o[~kvnan])
    assert torch.all((rows_g[kvnan] & 0x7F) == 0x7F)


@pytest.mark.parametrize("force", FORCE[1:])
def test_every_bf16_pattern_copies_bit_for_bit(force):
    w = W.make("copy", 8, 16, 0, seed=4, num_blocks=1, block_size=16)
    u = _all_bf16_patterns()
    w.q_nope.view(torch.int16).copy_(u.view(8, 16, 512))
    w.kv_c.view(torch.int16).copy_(u[-8 * 512:].view(8, 512))
    check_workload(w, extra_flags=force)


DIV_SCALES = [0.05, 1.0, 0.37, 3.0, 7.0, 0.9, 1.0 / 3.0, 2.0 ** -64, 2.0 ** 64, 1.9999999,
              1.0000001, 5e-20, 3e19, 448.0, 1e-3, 123.456]


@pytest.mark.parametrize("scale", DIV_SCALES)
def test_quotient_equals_ieee_division_for_every_fp32(scale):
    """The epilogue's x / scale against CUDA's IEEE division for all 2^32 fp32
    bit patterns: the same e4m3 byte everywhere (as fp32, and each half as
    bf16), and the same quotient bits for 2^-100 <= |x| and |x / scale| < 448
    (NaN counted equal)."""
    res = torch.zeros(3, dtype=torch.int64, device="cuda")
    rc = E.mla_harness_div_check(scale, 0, 2 ** 32, res.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == E.MLA_OK
    bad_q, bad_b, first = res.cpu().tolist()
    assert (bad_q, bad_b) == (0, 0), f"scale {scale}: {bad_q} quotients, {bad_b} bytes differ, first 0x{first & 0xffffffff:08x}"


# every scale significand of a binade: 2^23 scales x 65536 bf16 values each;
# the edges of the fast range, the bench's 0.05 (binade -5) and a few others
BF16_SCALE_BINADES = [-64, -9, -5, 0, 10, 63]


@pytest.mark.parametrize("e", BF16_SCALE_BINADES)
def test_bf16_bytes_equal_ieee_division_for_every_scale_of_a_binade(e):
    """The e4m3 byte of every bf16 value divided by every fp32 scale in
    [2^e, 2^(e+1)) equals the byte of CUDA's IEEE quotient (the epilogue's
    bf16 quotient takes one corrected step, exact in e4m3 but not in fp32)."""
    first = (e + 127) << 23
    res = torch.zeros(2, dtype=torch.int64, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    chunk = 1 << 21
    for c in range((1 << 23) // chunk):
        rc = E.mla_harness_bf16_scale_check(first + c * chunk, chunk, res.data_ptr(), stream)
        assert rc == E.MLA_OK
        bad, lowest = res.cpu().tolist()
        assert bad == 0, f"{bad} bytes differ, first at scale 0x{lowest & 0xffffffff:08x}"


# ---- edge cases

def test_zero_tokens_touches_nothing():
    w = W.make("empty", 0, 4, W.FLAG_ROPE, seed=1, num_blocks=1, rope_rows=8, cache_fill="random")
    d = w.to("cuda")
    q = torch.empty((0, 4, 576), dtype=torch.bfloat16, device="cuda")
    before = d.cache.clone()
    assert E.launch_workload(d, q) == E.MLA_OK
    torch.cuda.synchronize()
    assert torch.equal(d.cache.view(torch.int16), before.view(torch.int16))


@pytest.mark.parametrize("force", FORCE)
def test_bad_slots_and_positions(force):
    w = W.make("rules", 40, 3, W.FLAG_ROPE | W.FLAG_KV_FP8, seed=9, num_blocks=2, block_size=32,
               cache_fill="random", rope_rows=16)
    w.slot_mapping[1] = -1
    w.slot_mapping[2] = 64            # == capacity
    w.slot_mapping[5] = 2 ** 40       # far out
    w.positions[3] = 16               # == rope_rows
    w.positions[4] = -5
    w.positions[7] = 2 ** 31 - 1
    qg, cg, sg = run_gpu(w, extra_flags=force)
    qo, co, so = run_oracle(w)
    assert sg == so == E.MLA_STATUS_SLOT_RANGE | E.MLA_STATUS_POS_RANGE
    assert_same(qg, qo, "q_out")
    assert_same(cg, co, "cache")


@pytest.mark.parametrize("force", FORCE)
def test_one_token_one_head_and_max_heads(force):
    for T, H in ((1, 1), (1, 128), (2, 1024)):
        w = W.make("tiny", T, H, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=T + H, num_blocks=1, block_size=8,
                   rope_rows=64, scale=0.05, cache_fill="random")
        check_workload(w, extra_flags=force)


@pytest.mark.parametrize("force", FORCE[1:])
@pytest.mark.parametrize("T,H", [(2, 65536), (3, 40009)])
def test_largest_head_counts(force, T, H):
    """The head count limit and a large odd one: (token, head) come from the
    row index by a multiply-high division, exact over every row of a call."""
    w = W.make("many_heads", T, H, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=T + H, num_blocks=1, block_size=8,
               rope_rows=64, scale=0.05, cache_fill="random")
    check_workload(w, extra_flags=force)


def test_misaligned_arguments_launch_nothing():
    w = W.make("align", 4, 4, 0, seed=2, num_blocks=1, cache_fill="random")
    d = w.to("cuda")
    q = torch.zeros((4, 4, 576), dtype=torch.bfloat16, device="cuda")
    before = d.cache.clone()
    base = dict(q_nope=d.q_nope.data_ptr(), q_nope_stride_t=d.q_nope.stride(0),
                q_nope_stride_h=d.q_nope.stride(1), q_pe=d.q_pe.data_ptr(), q_pe_stride_t=d.q_pe.stride(0),
                q_pe_stride_h=d.q_pe.stride(1), kv_c=d.kv_c.data_ptr(), kv_c_stride_t=d.kv_c.stride(0),
                k_pe=d.k_pe.data_ptr(), k_pe_stride_t=d.k_pe.stride(0), slot_mapping=d.slot_mapping.data_ptr(),
                positions=None, cos_sin=None, rope_rows=0, q_scale=None, kv_scale=None, T=4, H=4,
                block_size=64, num_blocks=1, flags=0, q_out=q.data_ptr(), cache=d.cache.data_ptr(),
                status=None, stream=torch.cuda.current_stream().cuda_stream)
    for k, off in (("q_nope", 2), ("kv_c", 8), ("q_out", 2), ("cache", 4)):
        args = dict(base)
        args[k] += off
        assert E.mla_epilogue_launch(**args) == E.MLA_ERR_ALIGNMENT
    torch.cuda.synchronize()
    assert torch.equal(d.cache.view(torch.int16), before.view(torch.int16)) and torch.count_nonzero(q) == 0
    assert E.mla_epilogue_launch(**base) == E.MLA_OK
    torch.cuda.synchronize()
    assert torch.count_nonzero(q) > 0


# ---- programmatic dependent launch behind the synthetic producer

@pytest.mark.parametrize("force", FORCE)
def test_pdl_behind_producer_repeated(force):
    """Several producer -> epilogue(PDL) rounds on one stream with fresh data
    each time: a query row that read before the producer finished would see
    zeros or the previous round's values."""
    for rnd in range(3):
        w = W.make("pdl", 300, 16, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=50 + rnd,
                   num_blocks=64, rope_rows=4096, scale=0.05, cache_fill="random")
        check_workload(w, extra_flags=force, producer=True)


def test_torch_convenience_wrapper_matches_oracle():
    w = W.make("wrap", 9, 16, W.FLAG_ROPE | W.FLAG_KV_FP8, seed=77, num_blocks=2, rope_rows=128,
               scale=0.05, cache_fill="random")
    d = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    q = E.fused_mla_decode_q_concat_kv_cache_insert(d.q_nope, d.q_pe, d.kv_c, d.k_pe, d.cache,
                                                    d.slot_mapping, positions=d.positions,
                                                    cos_sin=d.cos_sin, kv_scale=d.kv_scale, status=status)
    torch.cuda.synchronize()
    qo, co, so = run_oracle(w)
    assert_same(q.cpu(), qo, "q_out")
    assert_same(d.cache.cpu(), co, "cache")
    assert int(status.item()) == so == 0
    with pytest.raises(E.MlaError):
        E.fused_mla_decode_q_concat_kv_cache_insert(d.q_nope, d.q_pe, d.kv_c, d.k_pe, d.cache,
                                                    d.slot_mapping, positions=d.positions,
                                                    cos_sin=d.cos_sin, kv_scale=d.kv_scale,
                                                    extra_flags=E.MLA_FLAG_FORCE_ROWS | E.MLA_FLAG_FORCE_SPLIT)


@pytest.mark.parametrize("scale", [1e-25, 5e25, -0.5, 2.0 ** -70, 0.0, float("inf")])
@pytest.mark.parametrize("force", FORCE[1:])
def test_scales_outside_the_fast_range(scale, force):
    """Scales outside [2^-64, 2^64] (and zero, negative, infinite ones) take
    the IEEE-division path in both kernels: bytes equal the oracle's, NaN
    results compared as NaN (the sign of a NaN code is not specified)."""
    w = W.make("scales", 9, 16, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=12, num_blocks=1,
               block_size=16, std=3.0, rope_rows=64, cache_fill="random")
    w.q_scale.fill_(scale)
    w.kv_scale.fill_(scale)
    qg, cg, _ = run_gpu(w, extra_flags=force)
    qo, co, _ = run_oracle(w)
    for g, o, what in ((qg, qo, "q_out"), (cg, co, "cache")):
        nan = (o & 0x7F) == 0x7F
        assert torch.all((g[nan] & 0x7F) == 0x7F), what
        assert torch.equal(g[~nan], o[~nan]), what
